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

// Selection key of (value, expert): larger keys come first.  The float's bits are made monotonic
// as an unsigned integer (NaN is mapped to -inf before, -0 to +0), and the low half holds ~e, so
// equal values order by lower expert id: the tie rule of the selection.  Key 0 (below every real
// key) is "none".
__device__ __forceinline__ unsigned long long sel_key(float v, int e) {
  uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);   // -0 and +0 compare equal: one key
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<unsigned long long>(u) << 32) | static_cast<uint32_t>(~e);
}
__device__ __forceinline__ float key_value(unsigned long long key) {
  uint32_t u = static_cast<uint32_t>(key >> 32);
  u = (u & 0x80000000u) ? (u & 0x7fffffffu) : ~u;
  return __uint_as_float(u);
}
__device__ __forceinline__ int key_expert(unsigned long long key) {
  return static_cast<int>(~static_cast<uint32_t>(key));
}
__device__ __forceinline__ void cswap(unsigned long long& a, unsigned long long& b) {   // a >= b after
  const unsigned long long hi = a > b ? a : b, lo = a > b ? b : a;
  a = hi;
  b = lo;
}

// With parts != null the logits row is first formed from the split-K parts of the gate GEMM
// (sum in part order, then the bias: the same float operations as a separate reduce) and
// written out, so the logits take one pass instead of two.  Each lane sorts its VPT keys once
// (descending); the k rounds then take the warp maximum of the lanes' heads, and the lane that
// held it pops its head.
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
    unsigned long long key[VPT];
    bool nan_seen = false;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int e = lane + 32 * i;
      key[i] = 0ull;
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
        key[i] = sel_key(x, e);
      }
    }
    // descending sort of the lane's keys (odd-even transposition: VPT rounds)
#pragma unroll
    for (int r = 0; r < VPT; ++r)
#pragma unroll
      for (int i = r & 1; i + 1 < VPT; i += 2) cswap(key[i], key[i + 1]);
    unsigned long long pick = 0ull;
    for (int r = 0; r < k; ++r) {
      unsigned long long best = key[0];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
        best = other > best ? other : best;
      }
      if (key[0] == best) {   // keys are distinct per expert: exactly one lane pops
#pragma unroll
        for (int i = 0; i + 1 < VPT; ++i) key[i] = key[i + 1];
        key[VPT - 1] = 0ull;
      }
      if (lane == r) pick = best;
    }
    const float pick_v = key_value(pick);
    const int pick_e = key_expert(pick);
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
