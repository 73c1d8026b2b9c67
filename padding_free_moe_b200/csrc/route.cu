// Top-k softmax gate: one warp per token ([B] "5.4 MoE模型在分布式训练中的应用",
// 训练流程 step a; large top-k: reading notes 需求).
//
// Each lane holds ceil(E / 32) logits in registers.  k rounds of a warp-wide
// argmax under the order (value descending, index ascending) pick the experts;
// the weights are the softmax over the picked logits, computed in float32.
// A NaN logit ranks below every number (including -inf) and raises
// PFMOE_DEV_NONFINITE, as does a token whose largest logit is +inf or -inf
// (its weights are then undefined).
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace pfmoe {
namespace {

// Does (va, ea) come before (vb, eb) in selection order?  ea/eb == INT_MAX means "none".
__device__ __forceinline__ bool before(float va, int ea, float vb, int eb) {
  if (ea == INT_MAX) return false;
  if (eb == INT_MAX) return true;
  return va > vb || (va == vb && ea < eb);
}

// With parts != null the logits row is first formed from the split-K parts of the gate GEMM
// (sum in part order, then the bias: the same float operations as a separate reduce) and
// written out, so the logits take one pass instead of two.
template <int VPT>
__global__ void __launch_bounds__(256) topk_kernel(float* __restrict__ logits, const float* __restrict__ parts,
                                                   int nparts, const float* __restrict__ bias, int T, int E, int k,
                                                   int32_t* __restrict__ ids, float* __restrict__ w,
                                                   int32_t* err) {
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  const long long pstride = static_cast<long long>(T) * E;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += nwarps) {
    float* z = logits + static_cast<long long>(t) * E;
    float v[VPT];
    uint32_t taken = 0;
    bool nan_seen = false;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int e = lane + 32 * i;
      if (e < E) {
        float x;
        if (parts) {
          const float* pp = parts + static_cast<long long>(t) * E + e;
          x = pp[0];
          for (int sp = 1; sp < nparts; ++sp) x += pp[sp * pstride];
          if (bias) x += bias[e];
          z[e] = x;
        } else {
          x = z[e];
        }
        if (x != x) { nan_seen = true; x = -INFINITY; }
        v[i] = x;
      } else {
        v[i] = -INFINITY;
        taken |= 1u << i;
      }
    }
    float pick_v = -INFINITY;
    int pick_e = 0;
    for (int r = 0; r < k; ++r) {
      float bv = -INFINITY;
      int be = INT_MAX;
#pragma unroll
      for (int i = 0; i < VPT; ++i)
        if (!((taken >> i) & 1u) && before(v[i], lane + 32 * i, bv, be)) { bv = v[i]; be = lane + 32 * i; }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (before(ov, oe, bv, be)) { bv = ov; be = oe; }
      }
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
      if (lane == r) { pick_v = bv; pick_e = be; }
    }
    const float m = __shfl_sync(0xffffffffu, pick_v, 0);
    const float ex = lane < k ? expf(pick_v - m) : 0.f;
    const float sum = warp_sum(ex);
    if (lane < k) {
      ids[static_cast<long long>(t) * k + lane] = pick_e;
      w[static_cast<long long>(t) * k + lane] = ex / sum;
    }
    // A largest logit of +inf or -inf (every logit -inf or NaN) leaves the weights undefined.
    if ((__any_sync(0xffffffffu, nan_seen) || !isfinite(m)) && lane == 0) dev_error(err, PFMOE_DEV_NONFINITE);
  }
}

template <int VPT>
int launch_vpt(float* logits, const float* parts, int nparts, const float* bias, int T, int E, int k, int32_t* ids,
               float* w, int32_t* err, cudaStream_t s) {
  long long blocks = (static_cast<long long>(T) * 32 + 255) / 256;
  const long long cap = static_cast<long long>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  PFMOE_LAUNCH("route_topk", s,
               topk_kernel<VPT><<<static_cast<int>(blocks), 256, 0, s>>>(logits, parts, nparts, bias, T, E, k, ids, w,
                                                                         err));
  return PFMOE_OK;
}

}  // namespace

int launch_topk(float* logits, const float* parts, int nparts, const float* bias, int T, int E, int k, int32_t* ids,
                float* w, int32_t* err, cudaStream_t s) {
  if (E <= 32) return launch_vpt<1>(logits, parts, nparts, bias, T, E, k, ids, w, err, s);
  if (E <= 64) return launch_vpt<2>(logits, parts, nparts, bias, T, E, k, ids, w, err, s);
  if (E <= 128) return launch_vpt<4>(logits, parts, nparts, bias, T, E, k, ids, w, err, s);
  if (E <= 256) return launch_vpt<8>(logits, parts, nparts, bias, T, E, k, ids, w, err, s);
  if (E <= 512) return launch_vpt<16>(logits, parts, nparts, bias, T, E, k, ids, w, err, s);
  return launch_vpt<32>(logits, parts, nparts, bias, T, E, k, ids, w, err, s);
}

}  // namespace pfmoe
