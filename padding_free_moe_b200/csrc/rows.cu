// Row-movement kernels of the padding-free layer: dispatch (PFT.x), combine,
// combine backward, token-gradient gather-sum with the gate's backward, and a
// small transpose.  All are HBM-bound.
//
// Dispatch and the combine's backward move rows through shared memory with 1-D
// bulk copies (cp.async.bulk, the copy engine of each SM): dispatch loads a piece
// of a token row once and stores it to the token's k PFT rows straight from
// shared memory; the combine's backward loads dY and the k PFT row pieces of a
// token into a ring stage and reads both there.  The two gather-sums (combine,
// token gradient) keep their k row loads in registers instead: one warp per
// (token, column chunk), 16-byte vector loads, every warp access a coalesced
// 512-byte run of one row (BF16), all k loads of a lane in flight at once.  At
// d = 7168, k = 8 that measured faster than a staged ring, whose consumers wait
// on each stage while the register form keeps 8 loads per lane outstanding.
// Nothing uses atomics on data; every sum runs over the k slots in slot order,
// so results are deterministic.
#include "common.cuh"
#include "kernels.h"

namespace pfmoe {
namespace {

// --------------------------------------------------------------- bulk copies
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void bar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool bar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait (2 s of %globaltimer): false, with PFMOE_DEV_TIMEOUT set, if it gave up.
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, int32_t* err) {
  if (bar_try(bar, parity)) return true;
  unsigned long long t0;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  while (true) {
    if (bar_try(bar, parity)) return true;
    unsigned long long t1;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
    if (t1 - t0 > 2000000000ull) {
      dev_error(err, PFMOE_DEV_TIMEOUT);
      return false;
    }
  }
}
// global -> shared, completing on an mbarrier (both addresses 16-byte aligned, bytes a multiple of 16)
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}
// shared -> global, tracked by the issuing thread's bulk groups
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(reinterpret_cast<uint64_t>(dst)),
               "r"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// X-MoE article §2.1.2: PFT row r holds token row token_ids[r].  Computed token-major with bulk
// copies: one warp per CTA; lane 0 loads a piece of x[t] into a ring buffer and, once it has
// landed, stores it to the token's k rows pos[t, j] straight from shared memory.  Work items are
// (token, piece) pairs; DP_BUFS - 1 loads stay in flight, and a buffer is reloaded once the
// stores that read it have read it.
constexpr int DP_BUFS = 4;

__global__ void __launch_bounds__(32) dispatch_bulk_kernel(const char* __restrict__ x, const int32_t* __restrict__ pos,
                                                           int Tn, int k, int row_bytes, int piece_bytes, int pieces,
                                                           char* __restrict__ xp, int32_t* err) {
  extern __shared__ __align__(128) uint8_t dsm[];
  __shared__ __align__(8) uint64_t bar[DP_BUFS];
  const int lane = threadIdx.x;
  const long long N = static_cast<long long>(Tn) * k;
  const long long items = static_cast<long long>(Tn) * pieces;
  const long long first = blockIdx.x, stride = gridDim.x;
  if (first >= items) return;
  const long long n_my = (items - first + stride - 1) / stride;
  if (lane == 0) {
    for (int b = 0; b < DP_BUFS; ++b) bar_init(smem_addr(&bar[b]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  const uint32_t buf0 = smem_addr(dsm);
  auto piece_of = [&](long long i, long long& t, int& off, int& bytes) {
    const long long it = first + i * stride;
    t = it / pieces;
    const int c = static_cast<int>(it - t * pieces);
    off = c * piece_bytes;
    bytes = min(piece_bytes, row_bytes - off);
  };
  auto issue_load = [&](long long i) {
    long long t;
    int off, bytes;
    piece_of(i, t, off, bytes);
    const int b = static_cast<int>(i % DP_BUFS);
    const uint32_t bb = smem_addr(&bar[b]);
    bar_expect_tx(bb, bytes);
    bulk_load(buf0 + b * piece_bytes, x + t * row_bytes + off, bytes, bb);
  };
  if (lane == 0)
    for (long long i = 0; i < DP_BUFS - 1 && i < n_my; ++i) issue_load(i);
  bool ok = true;
  long long i = 0;
  for (; i < n_my && ok; ++i) {
    long long t;
    int off, bytes;
    piece_of(i, t, off, bytes);
    int my_pos = lane < k ? pos[t * k + lane] : 0;
    const bool bad = lane < k && (my_pos < 0 || my_pos >= N);
    const bool any_bad = __any_sync(0xffffffffu, bad);
    if (any_bad && lane == 0 && off == 0) dev_error(err, PFMOE_DEV_BAD_POS);
    const int b = static_cast<int>(i % DP_BUFS);
    ok = __all_sync(0xffffffffu, bar_wait(smem_addr(&bar[b]), static_cast<uint32_t>(i / DP_BUFS) & 1, err));
    if (!ok) break;
    for (int j = 0; j < k; ++j) {
      const long long pj = __shfl_sync(0xffffffffu, my_pos, j);
      if (lane == 0 && !any_bad) bulk_store(xp + pj * row_bytes + off, buf0 + b * piece_bytes, bytes);
    }
    if (lane == 0) {
      bulk_commit();
      // the next load goes into the buffer item i - 1 used: its stores (the group before this
      // one) must have read it
      if (i + DP_BUFS - 1 < n_my) {
        bulk_wait_read<1>();
        issue_load(i + DP_BUFS - 1);
      }
    }
    __syncwarp();
  }
  if (lane == 0) {
    // loads still in flight (after an abort) land before the CTA exits; stores complete
    for (long long r = i; r < n_my && r < i + DP_BUFS - 1; ++r)
      bar_wait(smem_addr(&bar[r % DP_BUFS]), static_cast<uint32_t>(r / DP_BUFS) & 1, err);
    bulk_wait_all();
  }
  __syncwarp();
}

// Consumer warps of the combine's backward: four per CTA, two CTAs per SM (measured faster than
// one CTA of eight consumer warps with larger pieces).
constexpr int GB_CONSUMERS = 128;
constexpr int GB_CWARPS = GB_CONSUMERS / 32;

// The combine's backward below runs a producer / consumer ring: warp 0 loads a work item's row
// pieces (piece bytes each) with bulk copies into a stage and posts the item's per-slot scalars
// there; four consumer warps (GB_CONSUMERS threads, one 16-byte vector each) read the stage.
// KM >= k bounds the per-thread slot arrays so they stay in registers.
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(GB_CONSUMERS) : "memory"); }
// Barrier of the consumer warps that also ANDs a flag over them: every consumer warp takes the
// same decision (to go on or to stop), so none is left waiting at a barrier another has left.
__device__ __forceinline__ bool consumers_all(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, %2, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "n"(GB_CONSUMERS)
      : "memory");
  return r != 0;
}

// Per token t (work items are its row pieces, in order): dO[pos[t, j]] = w[t, j] * dY[t] and
// g[t, j] = <dY[t], O[pos[t, j]]> (the combine's backward).  Stage: the dY piece, then the k O
// pieces.  Each consumer thread keeps its partial dot products over the token's pieces; after the
// last piece they are summed over the thread's warp and then over the consumer warps in order
// (deterministic).  A token with an out-of-range row index is flagged and left unwritten.
template <typename T, int KM>
__global__ void __launch_bounds__(32 + GB_CONSUMERS) combine_bwd_bulk_kernel(
    const char* __restrict__ dy, const char* __restrict__ O, const int32_t* __restrict__ pos,
    const float* __restrict__ w, int Tn, int k, int row_bytes, int piece, int pieces, int stages,
    char* __restrict__ dO, float* __restrict__ g, int32_t* err) {
  constexpr int VN = Vec<T>::n;
  extern __shared__ __align__(128) uint8_t csm[];
  __shared__ __align__(8) uint64_t full[8];
  __shared__ __align__(8) uint64_t empty[8];
  __shared__ int valid[8];
  __shared__ int spos[8][32];
  __shared__ float sw[8][32];
  __shared__ float red[GB_CWARPS][KM];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long N = static_cast<long long>(Tn) * k;
  const uint32_t stage_bytes = static_cast<uint32_t>(k + 1) * piece;
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      bar_init(smem_addr(&full[s]), 1);
      bar_init(smem_addr(&empty[s]), GB_CONSUMERS);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const uint32_t st0 = smem_addr(csm);
  if (warp == 0) {
    uint32_t pending = 0, pend_parity = 0;
    int q = 0;
    bool ok = true;
    for (long long t = blockIdx.x; t < Tn && ok; t += gridDim.x) {
      const int my_pos = lane < k ? pos[t * k + lane] : 0;
      const bool bad = lane < k && (my_pos < 0 || my_pos >= N);
      const bool any_bad = __any_sync(0xffffffffu, bad);
      const float my_w = lane < k ? w[t * k + lane] : 0.f;
      if (any_bad && lane == 0) dev_error(err, PFMOE_DEV_BAD_POS);
      for (int c = 0; c < pieces; ++c, ++q) {
        const int off = c * piece;
        const int bytes = min(piece, row_bytes - off);
        const int s = q % stages;
        const uint32_t ph = (q / stages) & 1;
        if (!__all_sync(0xffffffffu, bar_wait(smem_addr(&empty[s]), ph ^ 1, err))) { ok = false; break; }
        spos[s][lane] = my_pos;
        sw[s][lane] = my_w;
        if (lane == 0) valid[s] = any_bad ? 0 : 1;
        __syncwarp();
        const uint32_t fb = smem_addr(&full[s]);
        if (any_bad) {
          if (lane == 0) bar_arrive(fb);
          continue;
        }
        if (lane == 0) {
          bar_expect_tx(fb, static_cast<uint32_t>((k + 1) * bytes));
          pending |= 1u << s;
          pend_parity = (pend_parity & ~(1u << s)) | (ph << s);
          const uint32_t sb = st0 + s * stage_bytes;
          bulk_load(sb, dy + t * row_bytes + off, bytes, fb);
          for (int j = 0; j < k; ++j)
            bulk_load(sb + (j + 1) * piece, O + static_cast<long long>(spos[s][j]) * row_bytes + off, bytes, fb);
        }
        __syncwarp();
      }
    }
    if (lane == 0)
      for (int s = 0; s < stages; ++s)
        if (pending & (1u << s)) bar_wait(smem_addr(&full[s]), (pend_parity >> s) & 1, err);
    __syncwarp();
  } else {
    const int c16 = threadIdx.x - 32;
    const int cw = warp - 1;
    int q = 0;
    bool ok = true;
    for (long long t = blockIdx.x; t < Tn && ok; t += gridDim.x) {
      float part[KM];
#pragma unroll
      for (int j = 0; j < KM; ++j) part[j] = 0.f;
      bool tok_valid = true;
      for (int c = 0; c < pieces; ++c, ++q) {
        const int off = c * piece;
        const int bytes = min(piece, row_bytes - off);
        const int s = q % stages;
        if (!__all_sync(0xffffffffu, bar_wait(smem_addr(&full[s]), (q / stages) & 1, err))) { ok = false; break; }
        tok_valid = valid[s] != 0;
        if (tok_valid) {
          for (int v = c16; v * 16 < bytes; v += GB_CONSUMERS) {
            const uint8_t* sp = csm + s * stage_bytes + v * 16;
            float a[VN];
            load16(reinterpret_cast<const T*>(sp), a);
#pragma unroll
            for (int j = 0; j < KM; ++j) {
              if (j < k) {
                float o[VN], dv[VN];
                load16(reinterpret_cast<const T*>(sp + (j + 1) * piece), o);
                const float wj = sw[s][j];
#pragma unroll
                for (int i = 0; i < VN; ++i) {
                  part[j] = fmaf(a[i], o[i], part[j]);
                  dv[i] = a[i] * wj;
                }
                store16(reinterpret_cast<T*>(dO + static_cast<long long>(spos[s][j]) * row_bytes + off + v * 16), dv);
              }
            }
          }
        }
        bar_arrive(smem_addr(&empty[s]));
      }
      // every consumer warp takes these two barriers once per token and leaves with the others
#pragma unroll
      for (int j = 0; j < KM; ++j) {
        const float v = warp_sum(part[j]);
        if (lane == 0) red[cw][j] = v;
      }
      const bool all_ok = consumers_all(ok);   // red[] complete
      if (all_ok && tok_valid && c16 < k) {
        float gs = red[0][c16];
#pragma unroll
        for (int w = 1; w < GB_CWARPS; ++w) gs += red[w][c16];   // warps in order: deterministic
        g[t * k + c16] = gs;
      }
      consumers_sync();                        // red[] read before the next token writes it
      if (!all_ok) break;
    }
  }
}

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

// dz_{t, ids[t,j]} = w_j (g_j - sum_l w_l g_l) (zero elsewhere);
// dx[t] = sum_j dX_pft[pos[t, j]] + sum_j dz_j * Wg^T[ids[t, j]] (the second sum only when wgT is given).
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
    // The gate term; with wgT null the caller adds it afterwards (BF16: a tensor-core GEMM of the
    // dense dz rows against Wg^T that reduce-adds into dx).
    if (wgT != nullptr) {
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
  const int row_bytes = d * (dtype == PFMOE_BF16 ? 2 : 4);
  // pieces of at most 8 KB (multiples of 16 bytes), as even as the row allows
  const int pieces = (row_bytes + 8191) / 8192;
  const int piece_bytes = ((row_bytes + pieces - 1) / pieces + 15) & ~15;
  const long long items = static_cast<long long>(T) * pieces;
  long long grid = static_cast<long long>(num_sms()) * 8;
  if (grid > items) grid = items;
  const size_t smem = static_cast<size_t>(DP_BUFS) * piece_bytes;
  PFMOE_LAUNCH("dispatch", s,
               (dispatch_bulk_kernel<<<static_cast<int>(grid), 32, smem, s>>>(
                   static_cast<const char*>(x), pos, T, k, row_bytes, piece_bytes, pieces, static_cast<char*>(x_pft),
                   err)));
  return PFMOE_OK;
}


// Ring geometry for `slots` row pieces per stage: pieces of at most `piece_cap` bytes (smaller where
// fewer than three stages of them fit the CTA's `budget`), then as many stages of them as the
// budget holds (2 to 8), and how many such CTAs share an SM.  The copy engine's cost per copy
// favours large pieces; the consumers' share of the work per piece favours more CTAs per SM.
struct Ring {
  int piece, pieces, stages, ctas_per_sm;
  size_t smem;
};
static Ring ring_for(int row_bytes, int slots, int budget, int piece_cap) {
  Ring r;
  int cap = (budget / (3 * slots)) & ~15;
  if (cap < 16) cap = 16;
  r.piece = piece_cap < cap ? piece_cap : cap;
  if (r.piece > row_bytes) r.piece = row_bytes;     // row_bytes is a multiple of 16
  r.pieces = (row_bytes + r.piece - 1) / r.piece;
  const int stage = slots * r.piece;
  r.stages = budget / stage;
  if (r.stages > 8) r.stages = 8;
  if (r.stages < 2) r.stages = 2;
  r.smem = static_cast<size_t>(r.stages) * stage;
  r.ctas_per_sm = r.smem <= 100 * 1024 ? 2 : 1;
  return r;
}

template <typename T, int KM>
static int launch_cbwd_t(const void* dy, const void* out, const int32_t* pos, const float* w, int T_, int k,
                         int row_bytes, const Ring& r, int grid, void* dO, float* g, int32_t* err, cudaStream_t s) {
  PFMOE_TRY(smem_optin(reinterpret_cast<const void*>(&combine_bwd_bulk_kernel<T, KM>), 227 * 1024, "combine_bwd"));
  PFMOE_LAUNCH("combine_bwd", s,
               (combine_bwd_bulk_kernel<T, KM><<<grid, 32 + GB_CONSUMERS, r.smem, s>>>(
                   static_cast<const char*>(dy), static_cast<const char*>(out), pos, w, T_, k, row_bytes, r.piece,
                   r.pieces, r.stages, static_cast<char*>(dO), g, err)));
  return PFMOE_OK;
}

int launch_combine_bwd(const void* dy, const void* out, const int32_t* pos, const float* w, int T, int k, int d,
                       int dtype, void* dO, float* g, int32_t* err, cudaStream_t s) {
  const int row_bytes = d * (dtype == PFMOE_BF16 ? 2 : 4);
  const Ring r = ring_for(row_bytes, k + 1, 96 * 1024, 2048);
  long long grid = static_cast<long long>(num_sms()) * r.ctas_per_sm;
  if (grid > T) grid = T;
  const int gr = static_cast<int>(grid);
  if (dtype == PFMOE_BF16) {
    if (k <= 8) return launch_cbwd_t<__nv_bfloat16, 8>(dy, out, pos, w, T, k, row_bytes, r, gr, dO, g, err, s);
    if (k <= 16) return launch_cbwd_t<__nv_bfloat16, 16>(dy, out, pos, w, T, k, row_bytes, r, gr, dO, g, err, s);
    return launch_cbwd_t<__nv_bfloat16, 32>(dy, out, pos, w, T, k, row_bytes, r, gr, dO, g, err, s);
  }
  if (k <= 8) return launch_cbwd_t<float, 8>(dy, out, pos, w, T, k, row_bytes, r, gr, dO, g, err, s);
  if (k <= 16) return launch_cbwd_t<float, 16>(dy, out, pos, w, T, k, row_bytes, r, gr, dO, g, err, s);
  return launch_cbwd_t<float, 32>(dy, out, pos, w, T, k, row_bytes, r, gr, dO, g, err, s);
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
