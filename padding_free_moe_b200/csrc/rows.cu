// Row-movement kernels of the padding-free layer: dispatch (PFT.x), combine,
// combine backward, token-gradient gather-sum with the gate's backward, and a
// small transpose.  All are HBM-bound and move rows with 16-byte vector
// loads/stores, so every warp access is a coalesced 512-byte run of one row
// (BF16).  Dispatch gives a warp one token; the gather-sums give a warp one
// (token, column chunk) or one PFT row, which keeps many more row loads in
// flight.  Nothing uses atomics; every sum runs over the k slots in slot
// order, so results are deterministic.
#include "common.cuh"
#include "kernels.h"

namespace pfmoe {
namespace {

constexpr int WARPS = 8;   // warps per block

inline int token_grid(long long T) {
  long long b = (T + WARPS - 1) / WARPS;
  const long long cap = static_cast<long long>(num_sms()) * 16;
  if (b > cap) b = cap;
  return static_cast<int>(b < 1 ? 1 : b);
}

// Grid for `items` one-warp work items (grid-stride beyond 16 blocks of 8 warps per SM).
inline int item_grid(long long items) { return token_grid(items); }

// Lane j < k loads pos[t, j]; returns false (and flags) if any row index is out of range.
__device__ __forceinline__ bool load_pos(const int32_t* pos, long long t, int k, long long N, int lane, int& my_pos,
                                         int32_t* err) {
  my_pos = lane < k ? pos[t * k + lane] : 0;
  const bool bad = lane < k && (my_pos < 0 || my_pos >= N);
  if (__any_sync(0xffffffffu, bad)) {
    if (lane == 0) dev_error(err, PFMOE_DEV_BAD_POS);
    return false;
  }
  return true;
}

// X-MoE article §2.1.2: PFT row r holds token row token_ids[r].  Computed token-major:
// x[t] is read once and written to its k rows pos[t, j].
template <typename T, int U>
__global__ void __launch_bounds__(WARPS * 32) dispatch_kernel(const T* __restrict__ x, const int32_t* __restrict__ pos,
                                                              int Tn, int k, int d, T* __restrict__ xp, int32_t* err) {
  constexpr int VN = Vec<T>::n;
  const int lane = threadIdx.x & 31;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const long long N = static_cast<long long>(Tn) * k;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < Tn; t += nw) {
    int my_pos;
    if (!load_pos(pos, t, k, N, lane, my_pos, err)) continue;
    const T* src = x + static_cast<long long>(t) * d;
    for (int base = 0; base < d; base += 32 * VN * U) {   // warp-uniform trip count
      const int c0 = base + lane * VN;
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * 32 * VN;
        if (c < d) v[u] = __ldg(reinterpret_cast<const uint4*>(src + c));
      }
      for (int j = 0; j < k; ++j) {
        const long long p = __shfl_sync(0xffffffffu, my_pos, j);
        T* dst = xp + p * d;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int c = c0 + u * 32 * VN;
          if (c < d) *reinterpret_cast<uint4*>(dst + c) = v[u];
        }
      }
    }
  }
}

// The gather-sum kernels below take one work item per warp: a (token, column chunk) pair, the
// chunk being the 32 * VN columns one warp covers with one 16-byte vector per lane.  Every lane
// then has all k row loads of its chunk in flight at once, and a token's chunks sit on
// neighbouring warps (its pos / weight rows stay in L1).  Sums still run over the k slots in
// slot order with float32 accumulation, so results do not depend on the launch shape.
template <typename T>
__host__ __device__ inline int chunk_cols() { return 32 * Vec<T>::n; }

// Items per token when each item covers U column chunks.
__host__ __device__ inline int items_per_token(int d, int vn, int U) {
  const int C = (d + 32 * vn - 1) / (32 * vn);
  return (C + U - 1) / U;
}

// y[t] = sum_j w[t, j] * O[pos[t, j]].  An item covers U consecutive column chunks.
template <typename T, int U>
__global__ void __launch_bounds__(WARPS * 32) combine_kernel(const T* __restrict__ O, const int32_t* __restrict__ pos,
                                                             const float* __restrict__ w, int Tn, int k, int d,
                                                             T* __restrict__ y, int32_t* err) {
  constexpr int VN = Vec<T>::n;
  const int lane = threadIdx.x & 31;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const long long N = static_cast<long long>(Tn) * k;
  const int CU = items_per_token(d, VN, U);
  const long long items = static_cast<long long>(Tn) * CU;
  for (long long it = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; it < items; it += nw) {
    const long long t = it / CU;
    const int cb = static_cast<int>(it - t * CU) * U * chunk_cols<T>() + lane * VN;
    int my_pos;
    if (!load_pos(pos, t, k, N, lane, my_pos, err)) continue;
    const float my_w = lane < k ? w[t * k + lane] : 0.f;
    float acc[U][VN];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int i = 0; i < VN; ++i) acc[u][i] = 0.f;
#pragma unroll 8
    for (int j = 0; j < k; ++j) {
      const long long p = __shfl_sync(0xffffffffu, my_pos, j);
      const float wj = __shfl_sync(0xffffffffu, my_w, j);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c0 = cb + u * chunk_cols<T>();
        if (c0 < d) {
          float o[VN];
          load16(O + p * d + c0, o);
#pragma unroll
          for (int i = 0; i < VN; ++i) acc[u][i] = fmaf(wj, o[i], acc[u][i]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c0 = cb + u * chunk_cols<T>();
      if (c0 < d) store16(y + t * d + c0, acc[u]);
    }
  }
}

// One warp per PFT row r = (t, j): dO[pos[t, j]] = w[t, j] * dY[t];  g[t, j] = <dY[t], O[pos[t, j]]>.
template <typename T>
__global__ void __launch_bounds__(WARPS * 32) combine_bwd_kernel(const T* __restrict__ dy, const T* __restrict__ O,
                                                                 const int32_t* __restrict__ pos,
                                                                 const float* __restrict__ w, int Tn, int k, int d,
                                                                 T* __restrict__ dO, float* __restrict__ g,
                                                                 int32_t* err) {
  constexpr int VN = Vec<T>::n;
  const int lane = threadIdx.x & 31;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const long long N = static_cast<long long>(Tn) * k;
  for (long long r = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < N; r += nw) {
    const long long t = r / k;
    const long long p = pos[r];
    if (p < 0 || p >= N) {
      if (lane == 0) dev_error(err, PFMOE_DEV_BAD_POS);
      continue;
    }
    const float wj = w[r];
    const T* dyr = dy + t * d;
    const T* orow = O + p * d;
    T* drow = dO + p * d;
    float part = 0.f;
#pragma unroll 2
    for (int c0 = lane * VN; c0 < d; c0 += 32 * VN) {
      float a[VN], o[VN];
      load16(dyr + c0, a);
      load16(orow + c0, o);
#pragma unroll
      for (int i = 0; i < VN; ++i) {
        part = fmaf(a[i], o[i], part);
        a[i] *= wj;
      }
      store16(drow + c0, a);
    }
    part = warp_sum(part);
    if (lane == 0) g[r] = part;
  }
}

// dz_{t, ids[t,j]} = w_j (g_j - sum_l w_l g_l) (zero elsewhere);
// dx[t] = sum_j dX_pft[pos[t, j]] + sum_j dz_j * Wg^T[ids[t, j]].
// The dense dlogits row (and its BF16 copy for the dWg GEMM) is written by the token's chunk-0 item.
template <typename T, int U>
__global__ void __launch_bounds__(WARPS * 32) token_grad_kernel(const T* __restrict__ dxp, const int32_t* __restrict__ pos,
                                                                const float* __restrict__ g, const float* __restrict__ w,
                                                                const int32_t* __restrict__ ids,
                                                                const T* __restrict__ wgT, int Tn, int k, int d, int E,
                                                                T* __restrict__ dx, float* __restrict__ dlogits,
                                                                __nv_bfloat16* __restrict__ dz_bf16, int32_t* err) {
  constexpr int VN = Vec<T>::n;
  const int lane = threadIdx.x & 31;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  const long long N = static_cast<long long>(Tn) * k;
  const int CU = items_per_token(d, VN, U);
  const long long items = static_cast<long long>(Tn) * CU;
  for (long long it = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; it < items; it += nw) {
    const long long t = it / CU;
    const int ch = static_cast<int>(it - t * CU);
    const int cb = ch * U * chunk_cols<T>() + lane * VN;
    int my_pos;
    if (!load_pos(pos, t, k, N, lane, my_pos, err)) continue;
    const long long tk = t * k;
    const float my_w = lane < k ? w[tk + lane] : 0.f;
    const float my_g = lane < k ? g[tk + lane] : 0.f;
    int my_id = lane < k ? ids[tk + lane] : 0;
    if (lane < k && static_cast<unsigned>(my_id) >= static_cast<unsigned>(E)) {
      dev_error(err, PFMOE_DEV_BAD_EXPERT_ID);
      my_id = 0;
    }
    const float inner = warp_sum(my_w * my_g);
    const float my_dz = lane < k ? my_w * (my_g - inner) : 0.f;
    if (ch == 0) {
      for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        float val = 0.f;
        for (int j = 0; j < k; ++j) {
          const int idj = __shfl_sync(0xffffffffu, my_id, j);
          const float dzj = __shfl_sync(0xffffffffu, my_dz, j);
          if (idj == e) val = dzj;
        }
        if (e < E) {
          dlogits[t * E + e] = val;
          if (dz_bf16) dz_bf16[t * E + e] = __float2bfloat16_rn(val);
        }
      }
    }
    float acc[U][VN];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int i = 0; i < VN; ++i) acc[u][i] = 0.f;
#pragma unroll 8
    for (int j = 0; j < k; ++j) {
      const long long p = __shfl_sync(0xffffffffu, my_pos, j);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c0 = cb + u * chunk_cols<T>();
        if (c0 < d) {
          float v[VN];
          load16(dxp + p * d + c0, v);
#pragma unroll
          for (int i = 0; i < VN; ++i) acc[u][i] += v[i];
        }
      }
    }
#pragma unroll 8
    for (int j = 0; j < k; ++j) {
      const long long idj = __shfl_sync(0xffffffffu, my_id, j);
      const float dzj = __shfl_sync(0xffffffffu, my_dz, j);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c0 = cb + u * chunk_cols<T>();
        if (c0 < d) {
          float v[VN];
          load16(wgT + idj * d + c0, v);
#pragma unroll
          for (int i = 0; i < VN; ++i) acc[u][i] = fmaf(dzj, v[i], acc[u][i]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c0 = cb + u * chunk_cols<T>();
      if (c0 < d) store16(dx + t * d + c0, acc[u]);
    }
  }
}

template <typename T>
__global__ void transpose_kernel(const T* __restrict__ in, int rows, int cols, T* __restrict__ out) {
  __shared__ T tile[32][33];
  const int c = blockIdx.x * 32 + threadIdx.x;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int r = blockIdx.y * 32 + i;
    if (r < rows && c < cols) tile[i][threadIdx.x] = in[static_cast<long long>(r) * cols + c];
  }
  __syncthreads();
  const int r2 = blockIdx.y * 32 + threadIdx.x;
  for (int i = threadIdx.y; i < 32; i += 8) {
    const int c2 = blockIdx.x * 32 + i;
    if (c2 < cols && r2 < rows) out[static_cast<long long>(c2) * rows + r2] = tile[threadIdx.x][i];
  }
}

}  // namespace

int launch_dispatch(const void* x, const int32_t* pos, int T, int k, int d, int dtype, void* x_pft, int32_t* err,
                    cudaStream_t s) {
  const int g = token_grid(T);
  if (dtype == PFMOE_BF16) {
    PFMOE_LAUNCH("dispatch", s,
                 (dispatch_kernel<__nv_bfloat16, 4><<<g, WARPS * 32, 0, s>>>(
                     static_cast<const __nv_bfloat16*>(x), pos, T, k, d, static_cast<__nv_bfloat16*>(x_pft), err)));
  } else {
    PFMOE_LAUNCH("dispatch", s,
                 (dispatch_kernel<float, 4><<<g, WARPS * 32, 0, s>>>(static_cast<const float*>(x), pos, T, k, d,
                                                                     static_cast<float*>(x_pft), err)));
  }
  return PFMOE_OK;
}

// Column chunks per work item: one for rows of up to 16 chunks (d <= 4096 BF16), else 4, which
// keeps the per-token prologue (pos / weight loads, dlogits row) off wide rows.
static int chunks_per_item(int d, int vn) { return (d + 32 * vn - 1) / (32 * vn) > 16 ? 4 : 1; }

int launch_combine(const void* out, const int32_t* pos, const float* w, int T, int k, int d, int dtype, void* y,
                   int32_t* err, cudaStream_t s) {
  const int vn = dtype == PFMOE_BF16 ? 8 : 4;
  const int U = chunks_per_item(d, vn);
  const int g = item_grid(static_cast<long long>(T) * items_per_token(d, vn, U));
  if (dtype == PFMOE_BF16) {
    const auto* o = static_cast<const __nv_bfloat16*>(out);
    auto* yy = static_cast<__nv_bfloat16*>(y);
    if (U == 4) PFMOE_LAUNCH("combine", s, (combine_kernel<__nv_bfloat16, 4><<<g, WARPS * 32, 0, s>>>(o, pos, w, T, k, d, yy, err)));
    else PFMOE_LAUNCH("combine", s, (combine_kernel<__nv_bfloat16, 1><<<g, WARPS * 32, 0, s>>>(o, pos, w, T, k, d, yy, err)));
  } else {
    const auto* o = static_cast<const float*>(out);
    auto* yy = static_cast<float*>(y);
    if (U == 4) PFMOE_LAUNCH("combine", s, (combine_kernel<float, 4><<<g, WARPS * 32, 0, s>>>(o, pos, w, T, k, d, yy, err)));
    else PFMOE_LAUNCH("combine", s, (combine_kernel<float, 1><<<g, WARPS * 32, 0, s>>>(o, pos, w, T, k, d, yy, err)));
  }
  return PFMOE_OK;
}

int launch_combine_bwd(const void* dy, const void* out, const int32_t* pos, const float* w, int T, int k, int d,
                       int dtype, void* dO, float* g, int32_t* err, cudaStream_t s) {
  const int gr = item_grid(static_cast<long long>(T) * k);
  if (dtype == PFMOE_BF16) {
    PFMOE_LAUNCH("combine_bwd", s,
                 combine_bwd_kernel<__nv_bfloat16><<<gr, WARPS * 32, 0, s>>>(
                     static_cast<const __nv_bfloat16*>(dy), static_cast<const __nv_bfloat16*>(out), pos, w, T, k, d,
                     static_cast<__nv_bfloat16*>(dO), g, err));
  } else {
    PFMOE_LAUNCH("combine_bwd", s,
                 combine_bwd_kernel<float><<<gr, WARPS * 32, 0, s>>>(static_cast<const float*>(dy),
                                                                     static_cast<const float*>(out), pos, w, T, k, d,
                                                                     static_cast<float*>(dO), g, err));
  }
  return PFMOE_OK;
}

int launch_transpose(const void* in, int rows, int cols, int dtype, void* out, cudaStream_t s) {
  dim3 grid((cols + 31) / 32, (rows + 31) / 32), block(32, 8);
  if (dtype == PFMOE_BF16) {
    PFMOE_LAUNCH("transpose", s,
                 transpose_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(static_cast<const __nv_bfloat16*>(in), rows,
                                                                         cols, static_cast<__nv_bfloat16*>(out)));
  } else {
    PFMOE_LAUNCH("transpose", s,
                 transpose_kernel<float><<<grid, block, 0, s>>>(static_cast<const float*>(in), rows, cols,
                                                                static_cast<float*>(out)));
  }
  return PFMOE_OK;
}

int launch_token_grad(const void* dx_pft, const int32_t* pos, const float* g, const float* w, const int32_t* ids,
                      const void* wgT, int T, int k, int d, int E, int dtype, void* dx, float* dlogits,
                      void* dz_bf16, int32_t* err, cudaStream_t s) {
  const int vn = dtype == PFMOE_BF16 ? 8 : 4;
  const int U = chunks_per_item(d, vn);
  const int gr = item_grid(static_cast<long long>(T) * items_per_token(d, vn, U));
  auto* dzb = static_cast<__nv_bfloat16*>(dz_bf16);
  if (dtype == PFMOE_BF16) {
    const auto* a = static_cast<const __nv_bfloat16*>(dx_pft);
    const auto* wt = static_cast<const __nv_bfloat16*>(wgT);
    auto* o = static_cast<__nv_bfloat16*>(dx);
    if (U == 4)
      PFMOE_LAUNCH("token_grad", s, (token_grad_kernel<__nv_bfloat16, 4><<<gr, WARPS * 32, 0, s>>>(
                                         a, pos, g, w, ids, wt, T, k, d, E, o, dlogits, dzb, err)));
    else
      PFMOE_LAUNCH("token_grad", s, (token_grad_kernel<__nv_bfloat16, 1><<<gr, WARPS * 32, 0, s>>>(
                                         a, pos, g, w, ids, wt, T, k, d, E, o, dlogits, dzb, err)));
  } else {
    const auto* a = static_cast<const float*>(dx_pft);
    const auto* wt = static_cast<const float*>(wgT);
    auto* o = static_cast<float*>(dx);
    if (U == 4)
      PFMOE_LAUNCH("token_grad", s, (token_grad_kernel<float, 4><<<gr, WARPS * 32, 0, s>>>(
                                         a, pos, g, w, ids, wt, T, k, d, E, o, dlogits, dzb, err)));
    else
      PFMOE_LAUNCH("token_grad", s, (token_grad_kernel<float, 1><<<gr, WARPS * 32, 0, s>>>(
                                         a, pos, g, w, ids, wt, T, k, d, E, o, dlogits, dzb, err)));
  }
  return PFMOE_OK;
}

}  // namespace pfmoe
