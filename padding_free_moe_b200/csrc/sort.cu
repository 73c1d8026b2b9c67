// Stable counting sort by small integer keys, and the two index structures
// built on it: the padding-free token buffer (X-MoE article §2.1.1 "PFT数据结构创新")
// and the redundancy-bypassing-dispatch pilot plan (§2.2.1 "分层冗余消除算法").
//
// Sort = three launches over chunks of W * 256 consecutive keys (one CTA of W warps
// per chunk, W = 8 unless the per-warp counters would not fit in shared memory):
//   1. chunk histograms counts[c][key];
//   2. scan in (key, chunk) order -> per-key totals, key offsets and every chunk's base
//      row for every key (plus the grouped-GEMM tile prefix): one CTA for few chunks, else
//      a CTA per strip of keys, the last of which scans the key totals;
//   3. scatter: warp w of a chunk owns keys [256w, 256w + 256) of it; the warps count
//      their keys per key, take an exclusive prefix over warps, then walk their keys in
//      order, 32 at a time; lanes holding the same key find each other (one ballot per
//      key bit, or __match_any_sync for wide keys) and take consecutive rows in lane
//      order -> the sort is stable.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace pfmoe {
namespace {

constexpr int SCAN_THREADS = 1024;

constexpr int KPW = 256;   // keys per warp of a chunk (8 per lane)

// Warps per chunk CTA: up to 8, while the scatter's per-warp counters (W * K ints) fit in 48 KB.
inline int warps_per_block(int K) {
  int w = 12288 / (K > 0 ? K : 1);
  return w < 1 ? 1 : (w > 8 ? 8 : w);
}
inline long long chunk_keys(int K) { return static_cast<long long>(warps_per_block(K)) * KPW; }

__device__ __forceinline__ long long dev_count(long long n, const int32_t* n_dev) {
  return n_dev ? static_cast<long long>(*n_dev) : n;
}

// One CTA per chunk: shared histogram of the chunk's keys -> counts[chunk][key].
// It also zeroes the strip scan's ticket counter.
__global__ void chunk_hist_kernel(const int32_t* __restrict__ keys, long long n, const int32_t* n_dev, int K,
                                  int nchunks, int32_t* __restrict__ counts, unsigned* ticket, int32_t* err) {
  extern __shared__ int32_t sh[];
  const int chunk = blockIdx.x;
  if (chunk == 0 && threadIdx.x == 0) *ticket = 0u;
  for (int i = threadIdx.x; i < K; i += blockDim.x) sh[i] = 0;
  __syncthreads();
  const long long nn = dev_count(n, n_dev);
  const long long b = static_cast<long long>(chunk) * blockDim.x / 32 * KPW;
  // a chunk is blockDim.x * IT keys: every load of the thread is issued before its first atomic
  // (16-byte vectors for a whole chunk of 16-byte aligned keys)
  constexpr int IT = KPW / 32;
  int key[IT];
  const bool whole = b + static_cast<long long>(blockDim.x) * IT <= nn;
  if (whole && (reinterpret_cast<uintptr_t>(keys) & 15) == 0) {
    const int4* kv = reinterpret_cast<const int4*>(keys + b);
#pragma unroll
    for (int h = 0; h < IT / 4; ++h) {
      const int4 q = kv[h * blockDim.x + threadIdx.x];
      key[4 * h] = q.x;
      key[4 * h + 1] = q.y;
      key[4 * h + 2] = q.z;
      key[4 * h + 3] = q.w;
    }
  } else {
#pragma unroll
    for (int it = 0; it < IT; ++it) {
      const long long i = b + static_cast<long long>(it) * blockDim.x + threadIdx.x;
      key[it] = i < nn ? keys[i] : 0;
    }
  }
  bool bad = false;
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    if (!whole && b + static_cast<long long>(it) * blockDim.x + threadIdx.x >= nn) break;
    if (static_cast<unsigned>(key[it]) < static_cast<unsigned>(K)) atomicAdd(&sh[key[it]], 1);
    else bad = true;
  }
  if (bad) dev_error(err, PFMOE_DEV_BAD_EXPERT_ID);
  __syncthreads();
  if (chunk < nchunks)
    for (int i = threadIdx.x; i < K; i += blockDim.x) counts[static_cast<long long>(chunk) * K + i] = sh[i];
}

// Block-wide exclusive scan of one int per thread; returns the exclusive prefix, *total = block sum.
__device__ int block_excl_scan(int v, int* tmp /*[32]*/, int* total) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) tmp[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = lane < nw ? tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    tmp[lane] = s;  // inclusive warp sums
  }
  __syncthreads();
  const int warp_off = wid > 0 ? tmp[wid - 1] : 0;
  *total = tmp[nw - 1];
  __syncthreads();
  return warp_off + x - v;
}

// counts [C][K] -> totals [K], offsets [K+1], base [C][K] = rows of key k in chunks before c (relative
// to the key's first row; the scatter adds offsets[k]); optional tiles [K+1] = prefix of
// ceil(total/tile_rows).  One CTA: used while C is small (launch latency dominates there).
__global__ void __launch_bounds__(SCAN_THREADS) chunk_scan_kernel(const int32_t* __restrict__ counts, int C, int K,
                                                                  int32_t* totals, int32_t* offsets,
                                                                  int32_t* __restrict__ base, int32_t* tiles,
                                                                  int tile_rows) {
  __shared__ int tmp[32];
  int carry = 0, tcarry = 0;
  for (int k0 = 0; k0 < K; k0 += SCAN_THREADS) {
    const int key = k0 + threadIdx.x;
    int tot = 0;
    if (key < K)
      for (int c = 0; c < C; ++c) tot += counts[static_cast<long long>(c) * K + key];
    int blk;
    const int excl = block_excl_scan(tot, tmp, &blk) + carry;
    int tblk;
    const int nt = tile_rows > 0 ? (tot + tile_rows - 1) / tile_rows : 0;
    const int texcl = block_excl_scan(nt, tmp, &tblk) + tcarry;
    if (key < K) {
      if (totals) totals[key] = tot;
      offsets[key] = excl;
      if (tiles) tiles[key] = texcl;
      int run = 0;
      for (int c = 0; c < C; ++c) {
        const long long idx = static_cast<long long>(c) * K + key;
        const int cnt = counts[idx];
        base[idx] = run;
        run += cnt;
      }
    }
    carry += blk;
    tcarry += tblk;
  }
  if (threadIdx.x == 0) {
    offsets[K] = carry;
    if (tiles) tiles[K] = tcarry;
  }
}

// Key totals -> offsets [K+1], optional tiles [K+1] (prefix of ceil(total/tile_rows)), optional copy of
// totals: all threads of one CTA.  The totals are read from L2 (other CTAs wrote them).
__device__ void key_scan_body(const int32_t* totals, int K, int32_t* totals_out, int32_t* offsets, int32_t* tiles,
                              int tile_rows, int* tmp /*[32]*/) {
  int carry = 0, tcarry = 0;
  for (int k0 = 0; k0 < K; k0 += blockDim.x) {
    const int key = k0 + threadIdx.x;
    const int tot = key < K ? __ldcg(totals + key) : 0;
    int blk, tblk;
    const int excl = block_excl_scan(tot, tmp, &blk) + carry;
    const int nt = tile_rows > 0 ? (tot + tile_rows - 1) / tile_rows : 0;
    const int texcl = block_excl_scan(nt, tmp, &tblk) + tcarry;
    if (key < K) {
      if (totals_out) totals_out[key] = tot;
      offsets[key] = excl;
      if (tiles) tiles[key] = texcl;
    }
    carry += blk;
    tcarry += tblk;
  }
  if (threadIdx.x == 0) {
    offsets[K] = carry;
    if (tiles) tiles[K] = tcarry;
  }
}

// Many chunks: the [C][K] chunk counts scanned down their columns, for strips of STRIP_KEYS keys per
// CTA; its 32 warps take consecutive row segments, a warp instruction covering 32 / STRIP_KEYS rows of
// the strip.  Pass 1 sums each warp's segment per key, the segment sums are scanned per key across the
// warps, and pass 2 writes each element's exclusive prefix (relative base) in the same order.  A narrow
// strip spreads the scan over more SMs (K / STRIP_KEYS CTAs); the partly used sectors it reads are L2
// hits, the counts having just been written.  The last CTA to finish (a ticket counter that the
// histogram launch zeroed) turns the key totals into key offsets and tile offsets, which saves a launch.
constexpr int STRIP_KEYS = 2;
constexpr int STRIP_ROWS = 32 / STRIP_KEYS;   // rows per warp step

__global__ void __launch_bounds__(SCAN_THREADS) strip_scan_kernel(const int32_t* __restrict__ counts, int C, int K,
                                                                  int32_t* __restrict__ base, int32_t* totals,
                                                                  unsigned* ticket, int32_t* totals_out,
                                                                  int32_t* offsets, int32_t* tiles, int tile_rows) {
  __shared__ int wsum[SCAN_THREADS / 32][STRIP_KEYS];
  __shared__ int tmp[32];
  __shared__ bool last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kk = lane % STRIP_KEYS, rsub = lane / STRIP_KEYS;   // key of the strip, row of a step
  const int key = blockIdx.x * STRIP_KEYS + kk;
  const bool kok = key < K;
  const int R = (C + SCAN_THREADS / 32 - 1) / (SCAN_THREADS / 32);   // rows per warp
  const int r0 = min(C, warp * R), r1 = min(C, r0 + R);
  constexpr int U = 8;   // row steps whose loads are in flight together
  int sum = 0;
  for (int c0 = r0 + rsub; c0 < r1; c0 += STRIP_ROWS * U) {
    int v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + STRIP_ROWS * u;
      v[u] = kok && c < r1 ? counts[static_cast<long long>(c) * K + key] : 0;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) sum += v[u];
  }
#pragma unroll
  for (int o = STRIP_KEYS; o < 32; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (rsub == 0) wsum[warp][kk] = sum;
  __syncthreads();
  if (warp == 0 && lane < STRIP_KEYS) {
    int run = 0;
    for (int w = 0; w < SCAN_THREADS / 32; ++w) {
      const int x = wsum[w][lane];
      wsum[w][lane] = run;
      run += x;
    }
    if (blockIdx.x * STRIP_KEYS + lane < K) totals[blockIdx.x * STRIP_KEYS + lane] = run;
    __threadfence();   // the totals are visible to the CTA that takes the last ticket
  }
  __syncthreads();
  int carry = wsum[warp][kk];
  for (int c0 = r0; c0 < r1; c0 += STRIP_ROWS * U) {
    int v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + STRIP_ROWS * u + rsub;
      v[u] = c < r1 && kok ? counts[static_cast<long long>(c) * K + key] : 0;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + STRIP_ROWS * u + rsub;
      int x = v[u];   // inclusive prefix over the step's rows of this key (lanes kk, kk + STRIP_KEYS, ...)
#pragma unroll
      for (int o = 1; o < STRIP_ROWS; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o * STRIP_KEYS);
        if (rsub >= o) x += y;
      }
      if (c < r1 && kok) base[static_cast<long long>(c) * K + key] = carry + x - v[u];
      carry += __shfl_sync(0xffffffffu, x, (STRIP_ROWS - 1) * STRIP_KEYS + kk);
    }
  }
  if (threadIdx.x == 0) last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  key_scan_body(totals, K, totals_out, offsets, tiles, tile_rows, tmp);
  if (threadIdx.x == 0) *ticket = 0u;
}

// Stable scatter.  Pass 1 counts each warp's keys.  Pass 2 gives every element its sorted row p
// (its key's first row in this chunk, plus the rows of earlier warps with that key, plus its rank
// among the warp's equal keys) and stages it in shared memory in sorted order.  The write-out then
// stores the row-indexed outputs as runs of consecutive rows, so neighbouring lanes write
// neighbouring addresses instead of one scattered sector per element.
// Sink interface: preload(i) is read with the keys, before the passes (one int); at_source(i, p)
// writes the outputs indexed by element i; payload(i, pre, a, b) gives two ints carried to the sorted
// side; at_dest(p, key, a, b) writes the outputs indexed by row p.
// Lanes holding equal keys (peers) are found with __match_any_sync, or for keys of at most KEY_BITS
// bits with one ballot per key bit.
// Shared memory: [warps][K] counts, two [K] bases and three [warps * KPW] staging arrays.
__host__ __device__ inline size_t scatter_smem_bytes(int nw, int K) {
  return (static_cast<size_t>(nw) * K + 2 * static_cast<size_t>(K) + 3 * static_cast<size_t>(nw) * KPW) *
         sizeof(int32_t);
}

template <int KEY_BITS>
__device__ __forceinline__ unsigned key_peers(bool ok, int key) {
  const unsigned valid = __ballot_sync(0xffffffffu, ok);
  if constexpr (KEY_BITS == 0) {
    return __match_any_sync(0xffffffffu, ok ? key : -1 - static_cast<int>(threadIdx.x & 31)) & valid;
  } else {
    unsigned peers = valid;
#pragma unroll
    for (int bit = 0; bit < KEY_BITS; ++bit) {
      const bool set = (key >> bit) & 1;
      const unsigned bal = __ballot_sync(0xffffffffu, set);
      peers &= set ? bal : ~bal;
    }
    return peers;
  }
}

// Five blocks per SM (48 registers): the key, preload and peer registers of a thread's eight
// elements stay live across the passes; with 64 registers only four blocks fit, with 40 they spill.
template <class Sink, int KEY_BITS>
__global__ void __launch_bounds__(256, 5) chunk_scatter_kernel(const int32_t* __restrict__ keys, long long n, const int32_t* n_dev, int K,
                                     int nchunks, const int32_t* __restrict__ base,
                                     const int32_t* __restrict__ key_offsets, Sink sink) {
  extern __shared__ int32_t sh[];
  __shared__ int tmp[32];
  __shared__ int staged;
  const int nw = blockDim.x >> 5;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  int32_t* cnt = sh;                                   // [nw][K]: counts, then each warp's first staging slot
  int32_t* lbase = cnt + static_cast<long long>(nw) * K;   // [K]: first staging slot of each key
  int32_t* gbase = lbase + K;                          // [K]: first sorted row of each key in this chunk
  int32_t* skey = gbase + K;                           // [nw * KPW]: staged keys, in sorted order
  int32_t* spa = skey + nw * KPW;                      // staged payloads
  int32_t* spb = spa + nw * KPW;
  const long long nn = dev_count(n, n_dev);
  const long long b = (static_cast<long long>(chunk) * nw + w) * KPW;
  constexpr int IT = KPW / 32;
  // every global load of the CTA is issued here: the keys, the sink's preload, and the first row of
  // key threadIdx.x in this chunk
  int key[IT], pre[IT];
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const long long i = b + it * 32 + lane;
    key[it] = i < nn ? keys[i] : -1;
    pre[it] = i < nn ? sink.preload(i) : 0;
  }
  const int gfirst = threadIdx.x < K && chunk < nchunks
                         ? key_offsets[threadIdx.x] + base[static_cast<long long>(chunk) * K + threadIdx.x]
                         : 0;
  for (int i = threadIdx.x; i < nw * K; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  int32_t* wcnt = cnt + w * K;
  // pass 1: per-warp counts by shared atomics (a count does not depend on the order of equal keys)
#pragma unroll
  for (int it = 0; it < IT; ++it)
    if (static_cast<unsigned>(key[it]) < static_cast<unsigned>(K)) atomicAdd(&wcnt[key[it]], 1);
  __syncthreads();
  // per key: the run length in this chunk and its first row (a thread keeps its key's warp counts
  // in registers when it has one key)
  const bool one_key = K <= static_cast<int>(blockDim.x);
  int wc[8];   // nw <= 8
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    int run = 0;
#pragma unroll
    for (int w2 = 0; w2 < 8; ++w2)
      if (w2 < nw) {
        wc[w2] = cnt[w2 * K + k];
        run += wc[w2];
      }
    lbase[k] = run;
    gbase[k] = k == threadIdx.x ? gfirst
                                : (chunk < nchunks ? key_offsets[k] + base[static_cast<long long>(chunk) * K + k] : 0);
  }
  __syncthreads();
  // run lengths -> first staging slot of each key (exclusive scan over keys)
  int carry = 0;
  for (int k0 = 0; k0 < K; k0 += blockDim.x) {
    const int k = k0 + threadIdx.x;
    const int v = k < K ? lbase[k] : 0;
    int blk;
    const int ex = block_excl_scan(v, tmp, &blk);
    if (k < K) {
      lbase[k] = carry + ex;
      gbase[k] -= carry + ex;   // from here: sorted row - staging slot, for every slot of key k
    }
    carry += blk;
  }
  if (threadIdx.x == 0) staged = carry;
  // each warp's first staging slot of each key
  if (one_key) {
    if (static_cast<int>(threadIdx.x) < K) {
      int run = lbase[threadIdx.x];
#pragma unroll
      for (int w2 = 0; w2 < 8; ++w2)
        if (w2 < nw) {
          cnt[w2 * K + threadIdx.x] = run;
          run += wc[w2];
        }
    }
  } else {
    for (int k = threadIdx.x; k < K; k += blockDim.x) {
      int run = lbase[k];
      for (int w2 = 0; w2 < nw; ++w2) {
        const int c = cnt[w2 * K + k];
        cnt[w2 * K + k] = run;
        run += c;
      }
    }
  }
  __syncthreads();
  // pass 2: rows in key order within the warp; source-indexed outputs now, the rest staged
#pragma unroll
  for (int it = 0; it < IT; ++it) {
    const bool ok = static_cast<unsigned>(key[it]) < static_cast<unsigned>(K);
    const unsigned peers = key_peers<KEY_BITS>(ok, key[it]);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int c0 = ok ? wcnt[key[it]] : 0;
    __syncwarp();
    if (ok && rank == 0) wcnt[key[it]] = c0 + __popc(peers);
    __syncwarp();
    if (ok) {
      const long long i = b + it * 32 + lane;
      const int lp = c0 + rank;   // staging slot
      sink.at_source(i, gbase[key[it]] + lp);
      int32_t pa, pb;
      sink.payload(i, pre[it], pa, pb);
      skey[lp] = key[it];
      spa[lp] = pa;
      spb[lp] = pb;
    }
  }
  __syncthreads();
  // write-out in sorted order: consecutive slots of one key are consecutive rows
  const int nv = staged;
  for (int lp = threadIdx.x; lp < nv; lp += blockDim.x) {
    const int k = skey[lp];
    sink.at_dest(gbase[k] + lp, k, spa[lp], spb[lp]);
  }
}

// PFT: element i = (token i / k, slot i % k) of the t-major assignment list (N < 2^31).
struct PftSink {
  const float* w;
  int k;
  unsigned long long kinv;   // 2^64 / k rounded up (k > 1): i / k = high word of i * kinv for any 32-bit i
  int32_t* pos;
  int32_t* token_ids;
  int32_t* expert_ids;
  float* cw;
  __device__ int32_t preload(long long i) const { return __float_as_int(w[i]); }
  __device__ void at_source(long long i, int p) const { pos[i] = p; }
  __device__ void payload(long long i, int32_t pre, int32_t& a, int32_t& b) const {
    a = k > 1 ? static_cast<int32_t>(__umul64hi(static_cast<unsigned long long>(i), kinv)) : static_cast<int32_t>(i);
    b = pre;
  }
  __device__ void at_dest(int p, int key, int32_t a, int32_t b) const {
    token_ids[p] = a;
    expert_ids[p] = key;
    cw[p] = __int_as_float(b);
  }
};

// Single-CTA exclusive scan of n (device or host count) ints: out[0..n], out[n] = sum.
__global__ void __launch_bounds__(SCAN_THREADS) excl_scan_kernel(const int32_t* __restrict__ in, long long n,
                                                                 const int32_t* n_dev, int32_t* __restrict__ out) {
  __shared__ int tmp[32];
  const long long nn = dev_count(n, n_dev);
  int carry = 0;
  for (long long i0 = 0; i0 < nn; i0 += SCAN_THREADS) {
    const long long i = i0 + threadIdx.x;
    const int v = i < nn ? in[i] : 0;
    int blk;
    const int ex = block_excl_scan(v, tmp, &blk);
    if (i < nn) out[i] = carry + ex;
    carry += blk;
  }
  if (threadIdx.x == 0) out[nn] = carry;
}

// Long scans (tokens, pilots): three launches instead of one CTA walking the whole array.
//   tile_sum: per 8192-element tile, the sums of a (and of b);
//   tile_offsets: one CTA scans the tile sums in place and writes the totals;
//   tile_scan: each tile's exclusive scan plus its offset (each thread scans 8 consecutive values).
constexpr int TILE_PT = 8;
constexpr int SCAN_TILE = SCAN_THREADS * TILE_PT;

__global__ void __launch_bounds__(SCAN_THREADS) tile_sum_kernel(const int32_t* __restrict__ a,
                                                                const int32_t* __restrict__ b, long long n,
                                                                const int32_t* n_dev, int32_t* sum_a, int32_t* sum_b) {
  __shared__ int tmp[32];
  const long long nn = dev_count(n, n_dev);
  const long long t0 = static_cast<long long>(blockIdx.x) * SCAN_TILE;
  int va = 0, vb = 0;
#pragma unroll
  for (int i = 0; i < TILE_PT; ++i) {
    const long long idx = t0 + threadIdx.x + static_cast<long long>(i) * SCAN_THREADS;
    if (idx < nn) {
      va += a[idx];
      if (b) vb += b[idx];
    }
  }
  int tot;
  block_excl_scan(va, tmp, &tot);
  if (threadIdx.x == 0) sum_a[blockIdx.x] = tot;
  if (b) {
    block_excl_scan(vb, tmp, &tot);
    if (threadIdx.x == 0) sum_b[blockIdx.x] = tot;
  }
}

// sum_a[0..ntiles) -> exclusive prefix in place; the sum goes to *total_a and/or to out_end[n] (n = the
// device count when n_dev is given); *total_b = sum of sum_b (if given).
__global__ void __launch_bounds__(SCAN_THREADS) tile_offsets_kernel(int32_t* sum_a, const int32_t* sum_b, int ntiles,
                                                                    int32_t* total_a, int32_t* total_b,
                                                                    int32_t* out_end, long long n,
                                                                    const int32_t* n_dev) {
  __shared__ int tmp[32];
  int carry = 0, bcarry = 0;
  for (int i0 = 0; i0 < ntiles; i0 += SCAN_THREADS) {
    const int i = i0 + threadIdx.x;
    const int v = i < ntiles ? sum_a[i] : 0;
    int blk;
    const int ex = block_excl_scan(v, tmp, &blk);
    if (i < ntiles) sum_a[i] = carry + ex;
    carry += blk;
    if (sum_b) {
      int bblk;
      block_excl_scan(i < ntiles ? sum_b[i] : 0, tmp, &bblk);
      bcarry += bblk;
    }
  }
  if (threadIdx.x == 0) {
    if (total_a) *total_a = carry;
    if (total_b) *total_b = bcarry;
    if (out_end) out_end[dev_count(n, n_dev)] = carry;
  }
}

__global__ void __launch_bounds__(SCAN_THREADS) tile_scan_kernel(const int32_t* __restrict__ a, long long n,
                                                                 const int32_t* n_dev,
                                                                 const int32_t* __restrict__ tile_off,
                                                                 int32_t* __restrict__ out) {
  __shared__ int tmp[32];
  const long long nn = dev_count(n, n_dev);
  const long long t0 = static_cast<long long>(blockIdx.x) * SCAN_TILE;
  if (t0 >= nn) return;   // uniform per CTA
  const long long i0 = t0 + static_cast<long long>(threadIdx.x) * TILE_PT;
  int v[TILE_PT];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < TILE_PT; ++i) {
    v[i] = i0 + i < nn ? a[i0 + i] : 0;
    sum += v[i];
  }
  int blk;
  int run = block_excl_scan(sum, tmp, &blk) + tile_off[blockIdx.x];
#pragma unroll
  for (int i = 0; i < TILE_PT; ++i) {
    if (i0 + i < nn) out[i0 + i] = run;
    run += v[i];
  }
}

// ------------------------------------------------------------------------- RBD
// Per token (a group of G lanes, G = 8, 16 or 32 >= k, so one warp serves 32 / G tokens; lane j < k
// of the group holds expert e_j): rank experts by (e, lane); a lane "leads" its node (device) when
// no earlier-ranked lane of the group shares it.
struct TokView {
  int e, node, dev;
  bool valid;
  bool node_lead, dev_lead;
  int node_rank;   // index of this lane's node among the token's distinct nodes (ascending)
  int within;      // rank of e among the token's experts on the same node
  int same_node;   // experts of this token on this lane's node
  int sub;         // lane index within the token's group
};

template <int G>
__device__ __forceinline__ TokView token_view(const int32_t* ids, long long t, bool tvalid, int k, int E, int epd,
                                              int epn, int32_t* err) {
  const int lane = threadIdx.x & 31;
  TokView v;
  v.sub = lane & (G - 1);
  v.valid = tvalid && v.sub < k;
  int e = v.valid ? ids[t * k + v.sub] : 0;
  if (v.valid && static_cast<unsigned>(e) >= static_cast<unsigned>(E)) {
    dev_error(err, PFMOE_DEV_BAD_EXPERT_ID);
    e = 0;
  }
  v.e = e;
  v.node = e / epn;
  v.dev = e / epd;
  int node_before = 0, dev_before = 0, within = 0, same = 0;
  for (int j = 0; j < k; ++j) {
    // the other lanes' node and device come by shuffle: no division inside the loop
    const int oe = __shfl_sync(0xffffffffu, e, j, G);
    const int onode = __shfl_sync(0xffffffffu, v.node, j, G);
    const int odev = __shfl_sync(0xffffffffu, v.dev, j, G);
    const bool earlier = oe < e || (oe == e && j < v.sub);
    if (onode == v.node) {
      ++same;
      if (earlier) { ++node_before; ++within; }
    }
    if (odev == v.dev && earlier) ++dev_before;
  }
  v.node_lead = v.valid && node_before == 0;
  v.dev_lead = v.valid && dev_before == 0;
  v.within = within;
  v.same_node = same;
  const unsigned gmask = G == 32 ? 0xffffffffu : ((1u << G) - 1u);
  const unsigned leads = (__ballot_sync(0xffffffffu, v.node_lead) >> (lane & ~(G - 1))) & gmask;
  int rank = 0;
  for (int j = 0; j < k; ++j) {
    const int onode = __shfl_sync(0xffffffffu, v.node, j, G);
    if (((leads >> j) & 1u) && onode < v.node) ++rank;
  }
  v.node_rank = rank;
  return v;
}

// Token of this lane's group, for grid-stride loops over groups of G lanes.
template <int G>
__device__ __forceinline__ long long group_token(long long step) {
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  return (warp + step) * (32 / G) + ((threadIdx.x & 31) / G);
}

template <int G>
__global__ void rbd_count_kernel(const int32_t* ids, int T, int k, int E, int epd, int epn, int32_t* ucount,
                                 int32_t* dcount, int32_t* err) {
  const int lane = threadIdx.x & 31;
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long step = 0;; step += nw) {
    const long long t = group_token<G>(step);
    if (__all_sync(0xffffffffu, t >= T)) break;
    const TokView v = token_view<G>(ids, t, t < T, k, E, epd, epn, err);
    const unsigned gmask = G == 32 ? 0xffffffffu : ((1u << G) - 1u);
    const int shift = lane & ~(G - 1);
    const int u = __popc((__ballot_sync(0xffffffffu, v.node_lead) >> shift) & gmask);
    const int dd = __popc((__ballot_sync(0xffffffffu, v.dev_lead) >> shift) & gmask);
    if (v.sub == 0 && t < T) { ucount[t] = u; dcount[t] = dd; }
  }
}

// Scan of per-token pilot counts; counts[0] = P, counts[1] = sum of distinct (token, device) pairs.
__global__ void __launch_bounds__(SCAN_THREADS) rbd_scan_kernel(const int32_t* ucount, const int32_t* dcount, int T,
                                                                int32_t* pilot_base, int32_t* counts) {
  __shared__ int tmp[32];
  int carry = 0, dcarry = 0;
  for (int i0 = 0; i0 < T; i0 += SCAN_THREADS) {
    const int i = i0 + threadIdx.x;
    const int u = i < T ? ucount[i] : 0;
    const int dd = i < T ? dcount[i] : 0;
    int blk, dblk;
    const int ex = block_excl_scan(u, tmp, &blk);
    block_excl_scan(dd, tmp, &dblk);
    if (i < T) pilot_base[i] = carry + ex;
    carry += blk;
    dcarry += dblk;
  }
  if (threadIdx.x == 0) { counts[0] = carry; counts[1] = dcarry; }
}

// Token-major pilot list: key = node, token, replica count.
template <int G>
__global__ void rbd_emit_kernel(const int32_t* ids, int T, int k, int E, int epd, int epn, const int32_t* pilot_base,
                                int32_t* pkey, int32_t* ptoken, int32_t* prc, int32_t* err) {
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long step = 0;; step += nw) {
    const long long t = group_token<G>(step);
    if (__all_sync(0xffffffffu, t >= T)) break;
    const TokView v = token_view<G>(ids, t, t < T, k, E, epd, epn, err);
    if (v.node_lead) {
      const int i = pilot_base[t] + v.node_rank;
      pkey[i] = v.node;
      ptoken[i] = static_cast<int32_t>(t);
      prc[i] = v.same_node;
    }
  }
}

struct RbdSink {
  const int32_t* ptoken;
  const int32_t* prc;
  int32_t* pilot_token;
  int32_t* pilot_node;
  int32_t* rc_sorted;
  int32_t* psorted;
  __device__ int32_t preload(long long i) const { return prc[i]; }
  __device__ void at_source(long long i, int p) const { psorted[i] = p; }
  __device__ void payload(long long i, int32_t pre, int32_t& a, int32_t& b) const {
    a = ptoken[i];
    b = pre;
  }
  __device__ void at_dest(int p, int key, int32_t a, int32_t b) const {
    pilot_token[p] = a;
    pilot_node[p] = key;
    rc_sorted[p] = b;
  }
};

template <int G>
__global__ void rbd_final_kernel(const int32_t* ids, int T, int k, int E, int epd, int epn,
                                 const int32_t* pilot_base, const int32_t* psorted, const int32_t* replica_offsets,
                                 int32_t* assign_pilot, int32_t* replica_expert, int32_t* pilot_device,
                                 int32_t* err) {
  const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
  for (long long step = 0;; step += nw) {
    const long long t = group_token<G>(step);
    if (__all_sync(0xffffffffu, t >= T)) break;
    const TokView v = token_view<G>(ids, t, t < T, k, E, epd, epn, err);
    if (v.valid) {
      const int q = psorted[pilot_base[t] + v.node_rank];
      assign_pilot[t * k + v.sub] = q;
      replica_expert[replica_offsets[q] + v.within] = v.e;
      if (v.within == 0) pilot_device[q] = v.dev;
    }
  }
}


// ------------------------------------------------ RBD plan for maps of at most 8 nodes
// Every configured device map has at most 8 nodes; for those the plan needs no sort.  The
// pilots of node n, in token order, are the tokens that route to n, so pilot (t, n) sits at
// node_offsets[n] + #{t' < t routing to n}, and its replicas at the node's replica offset +
// #{replicas on n of tokens t' < t}: per-node prefix counts over tokens.  Three launches, one
// thread per token:
//   rbd_fast_count: per 256-token tile, per node: tokens routing to it and replicas on it;
//   rbd_fast_scan:  per node, exclusive prefix over tiles; node offsets, totals, P;
//   rbd_fast_emit:  per token, the in-tile prefix by warp scans, then every output.
constexpr int RF_NODES = 8;
constexpr int RF_TILE = 256;

// Division of an expert id (< 2^16) by a divisor d < 2^16 as a multiply-high: with m = ceil(2^32 / d),
// floor(v m / 2^32) = floor(v / d) whenever v, d < 2^16 (the error v (m - 2^32 / d) / 2^32 stays below
// 1 / d).  Replaces the per-id integer divisions of the per-token kernels.
struct FastDiv {
  unsigned m;
  int d;
  __device__ __forceinline__ explicit FastDiv(int d_) : m(d_ > 1 ? 0xffffffffu / static_cast<unsigned>(d_) + 1u : 0u), d(d_) {}
  __device__ __forceinline__ int operator()(int v) const {
    return d > 1 ? static_cast<int>(__umulhi(static_cast<unsigned>(v), m)) : v;
  }
};

// The tile's ids are staged in shared memory with coalesced loads, one padded row of KM + 1 ints per
// token (row r holds token r's k ids), so that each thread's reads of its own row are free of bank
// conflicts for every k.
template <int KM>
__device__ __forceinline__ void rf_stage_rows(const int32_t* __restrict__ ids, int T, int k, int32_t* rows) {
  const long long base = static_cast<long long>(blockIdx.x) * RF_TILE * k;
  const long long end = static_cast<long long>(T) * k;
  const FastDiv row_of(k);
  int v[KM];
#pragma unroll
  for (int it = 0; it < KM; ++it) {
    const long long g = base + it * RF_TILE + threadIdx.x;
    v[it] = it < k && g < end ? ids[g] : 0;
  }
#pragma unroll
  for (int it = 0; it < KM; ++it)
    if (it < k) {
      const int i = it * RF_TILE + threadIdx.x;   // below RF_TILE * KM <= 2^13, so the division is exact
      const int r = row_of(i);
      rows[r * (KM + 1) + (i - r * k)] = v[it];
    }
  __syncthreads();
}

// The token's k ids, from its padded row of the staged tile, or, for k = KM and 16-byte aligned ids,
// straight from global memory as KM / 4 16-byte vectors: a warp's loads then cover its 32 tokens'
// ids contiguously, and the staging round trip through shared memory (and its barrier) is skipped.
template <int KM>
__device__ __forceinline__ bool rf_direct(const int32_t* ids, int k) {
  return k == KM && (reinterpret_cast<uintptr_t>(ids) & 15) == 0;
}

template <int KM>
__device__ __forceinline__ void rf_ids_direct(const int32_t* __restrict__ ids, long long t, bool valid, int (&v)[KM]) {
  const int4* src = reinterpret_cast<const int4*>(ids + t * KM);
#pragma unroll
  for (int q = 0; q < KM / 4; ++q) {
    const int4 x = valid ? src[q] : make_int4(0, 0, 0, 0);
    v[4 * q] = x.x;
    v[4 * q + 1] = x.y;
    v[4 * q + 2] = x.z;
    v[4 * q + 3] = x.w;
  }
}

template <int KM>
__device__ __forceinline__ void rf_ids_row(const int32_t* row, bool valid, int k, int (&v)[KM]) {
#pragma unroll
  for (int j = 0; j < KM; ++j) v[j] = valid && j < k ? row[j] : 0;
}

// The token's ids as sort keys id * 256 + slot (slots k .. KM - 1 and tokens past T hold INT_MAX).
// Ids outside [0, E) are flagged (when err is given) and read as 0.
template <int KM>
__device__ __forceinline__ void rf_keys(const int (&v)[KM], bool valid, int k, int E, int32_t* err, int (&key)[KM]) {
#pragma unroll
  for (int j = 0; j < KM; ++j) {
    int x = INT_MAX;
    if (valid && j < k) {
      int id = v[j];
      if (static_cast<unsigned>(id) >= static_cast<unsigned>(E)) {
        if (err) dev_error(err, PFMOE_DEV_BAD_EXPERT_ID);
        id = 0;
      }
      x = (id << 8) | j;
    }
    key[j] = x;
  }
}

// Keys in ascending order.  Node and device are monotone in the id, so each node's replicas then form
// one run of the sorted keys, in (id, slot) order, and the run's first key is the node's lowest id.
// Bitonic sorting network, unrolled over KM.
template <int KM>
__device__ __forceinline__ void rf_sort(int (&key)[KM]) {
#pragma unroll
  for (int size = 2; size <= KM; size <<= 1)
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
      for (int i = 0; i < KM; ++i) {
        const int p = i ^ stride;
        if (p > i) {
          const int lo = min(key[i], key[p]), hi = max(key[i], key[p]);
          const bool up = (i & size) == 0;
          key[i] = up ? lo : hi;
          key[p] = up ? hi : lo;
        }
      }
}

// The token's replicas per node, 8 bits per node (k <= 32 < 256; nodes < RF_NODES = 8).
template <int KM>
__device__ __forceinline__ unsigned long long rf_node_counts(const int (&key)[KM], const FastDiv& node_of) {
  unsigned long long cnt = 0;
#pragma unroll
  for (int s = 0; s < KM; ++s)
    if (key[s] != INT_MAX) cnt += 1ull << (8 * node_of(key[s] >> 8));
  return cnt;
}

__device__ __forceinline__ int rf_node_field(unsigned long long packed, int n) {
  return static_cast<int>((packed >> (8 * n)) & 0xffu);
}

// Packed per-node count of one token: bit 0..15 = 1 if the token routes to the node, 16..31 = its
// replicas there (sums over a 256-token tile stay below 2^16 in both fields).
__device__ __forceinline__ int rf_packed(unsigned long long cnt, int n) {
  const int r = rf_node_field(cnt, n);
  return (r > 0 ? 1 : 0) | (r << 16);
}

template <int KM>
__global__ void __launch_bounds__(RF_TILE) rbd_fast_count_kernel(const int32_t* __restrict__ ids, int T, int k, int E,
                                                                 int epd, int epn, int32_t* __restrict__ tile_cnt,
                                                                 int32_t* __restrict__ tile_dev, int32_t* err) {
  __shared__ int red[RF_TILE / 32][RF_NODES + 1];
  __shared__ int32_t rows[RF_TILE * (KM + 1)];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long t = static_cast<long long>(blockIdx.x) * RF_TILE + threadIdx.x;
  const bool valid = t < T;
  int v[KM];
  if (rf_direct<KM>(ids, k)) {
    rf_ids_direct<KM>(ids, t, valid, v);
  } else {
    rf_stage_rows<KM>(ids, T, k, rows);
    rf_ids_row<KM>(rows + threadIdx.x * (KM + 1), valid, k, v);
  }
  const FastDiv node_of(epn), dev_of(epd);
  int key[KM];
  rf_keys<KM>(v, valid, k, E, err, key);
  int dc = 0;   // distinct devices of the token
  if (E <= 64 * epd) {   // at most 64 devices: a bit per device, the ids need no order
    unsigned long long seen = 0;
#pragma unroll
    for (int s = 0; s < KM; ++s)
      if (key[s] != INT_MAX) seen |= 1ull << dev_of(key[s] >> 8);
    dc = __popcll(seen);
  } else {   // the device changes along the sorted ids
    rf_sort<KM>(key);
    int prev = -1;
#pragma unroll
    for (int s = 0; s < KM; ++s)
      if (key[s] != INT_MAX) {
        const int dv = dev_of(key[s] >> 8);
        dc += dv != prev;
        prev = dv;
      }
  }
  const unsigned long long cnt = rf_node_counts<KM>(key, node_of);
  // warp sums by the hardware reduction (the packed fields stay below 2^16: 32 flags, 32 k replicas)
#pragma unroll
  for (int n = 0; n < RF_NODES; ++n) {
    const int v = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(rf_packed(cnt, n))));
    if (lane == 0) red[warp][n] = v;
  }
  dc = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(dc)));
  if (lane == 0) red[warp][RF_NODES] = dc;
  __syncthreads();
  if (threadIdx.x <= RF_NODES) {
    int v = 0;
    for (int w = 0; w < RF_TILE / 32; ++w) v += red[w][threadIdx.x];
    if (threadIdx.x < RF_NODES) tile_cnt[static_cast<long long>(blockIdx.x) * RF_NODES + threadIdx.x] = v;
    else tile_dev[blockIdx.x] = v;
  }
}

// One CTA of 512 threads: thread i takes a run of RF_RUN consecutive tiles, the runs are scanned per
// node across the block, and each thread writes its tiles' exclusive token bases (in place) and
// replica bases (tile_rep_base); then the node offsets, P and the distinct (token, device) total.
// The [tile][node] rows go through shared memory: read and written with coalesced accesses, each
// thread's run of RF_RUN * RF_NODES ints padded by one int so that the per-thread reads are free of
// bank conflicts.  Tiles beyond one block's worth are handled in further passes.
constexpr int RF_SCAN_THREADS = 512;
constexpr int RF_RUN = 4;                              // tiles per thread per pass
constexpr int RF_ROW = RF_RUN * RF_NODES + 1;          // padded ints per thread run
constexpr int RF_SCAN_SMEM = 2 * RF_SCAN_THREADS * RF_ROW * 4;

__global__ void __launch_bounds__(RF_SCAN_THREADS) rbd_fast_scan_kernel(int ntiles, int n_nodes,
                                                                        int32_t* __restrict__ tile_cnt,
                                                                        int32_t* __restrict__ tile_rep_base,
                                                                        const int32_t* __restrict__ tile_dev,
                                                                        int32_t* pilots_per_node, int32_t* node_offsets,
                                                                        int32_t* node_rep_off, int32_t* counts,
                                                                        int32_t* replica_offsets) {
  extern __shared__ int32_t scan_sm[];
  int32_t* s_tok = scan_sm;                            // [thread][RF_ROW]: counts in, token bases out
  int32_t* s_rep = scan_sm + RF_SCAN_THREADS * RF_ROW; // replica bases out
  __shared__ int wt[RF_SCAN_THREADS / 32][RF_NODES], wr[RF_SCAN_THREADS / 32][RF_NODES];
  __shared__ int carry_t[RF_NODES], carry_r[RF_NODES];
  __shared__ int dsum[RF_SCAN_THREADS / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x < RF_NODES) { carry_t[threadIdx.x] = 0; carry_r[threadIdx.x] = 0; }
  int ds = 0;
  __syncthreads();
  for (int base = 0; base < ntiles; base += RF_SCAN_THREADS * RF_RUN) {
    const int nt = min(RF_SCAN_THREADS * RF_RUN, ntiles - base);   // tiles in this pass
    const long long g0 = static_cast<long long>(base) * RF_NODES;
    constexpr int PASS_INTS = RF_SCAN_THREADS * RF_RUN * RF_NODES;
    if (nt == RF_SCAN_THREADS * RF_RUN) {   // a whole pass: every load of the thread in flight at once
      int x[PASS_INTS / RF_SCAN_THREADS];
#pragma unroll
      for (int q = 0; q < PASS_INTS / RF_SCAN_THREADS; ++q) x[q] = tile_cnt[g0 + q * RF_SCAN_THREADS + threadIdx.x];
#pragma unroll
      for (int q = 0; q < PASS_INTS / RF_SCAN_THREADS; ++q) {
        const int i = q * RF_SCAN_THREADS + threadIdx.x;
        s_tok[(i / (RF_RUN * RF_NODES)) * RF_ROW + i % (RF_RUN * RF_NODES)] = x[q];
      }
    } else {
      for (int i = threadIdx.x; i < nt * RF_NODES; i += RF_SCAN_THREADS)
        s_tok[(i / (RF_RUN * RF_NODES)) * RF_ROW + i % (RF_RUN * RF_NODES)] = tile_cnt[g0 + i];
    }
    for (int i = threadIdx.x; i < nt; i += RF_SCAN_THREADS) ds += tile_dev[base + i];
    __syncthreads();
    const int t0 = base + threadIdx.x * RF_RUN;
    int v[RF_RUN][RF_NODES];
#pragma unroll
    for (int r = 0; r < RF_RUN; ++r) {
      const bool ok = t0 + r < ntiles;
#pragma unroll
      for (int n = 0; n < RF_NODES; ++n)
        v[r][n] = ok && n < n_nodes ? s_tok[threadIdx.x * RF_ROW + r * RF_NODES + n] : 0;
    }
    int run_t[RF_NODES], run_r[RF_NODES], ex_t[RF_NODES], ex_r[RF_NODES];
#pragma unroll
    for (int n = 0; n < RF_NODES; ++n) {
      run_t[n] = 0;
      run_r[n] = 0;
#pragma unroll
      for (int r = 0; r < RF_RUN; ++r) { run_t[n] += v[r][n] & 0xffff; run_r[n] += v[r][n] >> 16; }
      int a = run_t[n], b = run_r[n];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int ya = __shfl_up_sync(0xffffffffu, a, o);
        const int yb = __shfl_up_sync(0xffffffffu, b, o);
        if (lane >= o) { a += ya; b += yb; }
      }
      ex_t[n] = a - run_t[n];
      ex_r[n] = b - run_r[n];
      if (lane == 31) { wt[warp][n] = a; wr[warp][n] = b; }
    }
    __syncthreads();
    // warp totals -> warp offsets (warp 0, one lane per node), plus the carry from earlier passes
    if (warp == 0 && lane < RF_NODES) {
      int st = carry_t[lane], sr = carry_r[lane];
      for (int w = 0; w < RF_SCAN_THREADS / 32; ++w) {
        const int xt = wt[w][lane], xr = wr[w][lane];
        wt[w][lane] = st;
        wr[w][lane] = sr;
        st += xt;
        sr += xr;
      }
      carry_t[lane] = st;
      carry_r[lane] = sr;
    }
    __syncthreads();
#pragma unroll
    for (int n = 0; n < RF_NODES; ++n) {
      int at = wt[warp][n] + ex_t[n], ar = wr[warp][n] + ex_r[n];
#pragma unroll
      for (int r = 0; r < RF_RUN; ++r) {
        s_tok[threadIdx.x * RF_ROW + r * RF_NODES + n] = at;
        s_rep[threadIdx.x * RF_ROW + r * RF_NODES + n] = ar;
        at += v[r][n] & 0xffff;
        ar += v[r][n] >> 16;
      }
    }
    __syncthreads();
    // columns n >= n_nodes are written too (zero counts, so the bases repeat): the rows stay whole
    for (int i = threadIdx.x; i < nt * RF_NODES; i += RF_SCAN_THREADS) {
      const int si = (i / (RF_RUN * RF_NODES)) * RF_ROW + i % (RF_RUN * RF_NODES);
      tile_cnt[g0 + i] = s_tok[si];
      tile_rep_base[g0 + i] = s_rep[si];
    }
    __syncthreads();   // the buffers and wt / wr are rewritten by the next pass
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ds += __shfl_xor_sync(0xffffffffu, ds, o);
  if (lane == 0) dsum[warp] = ds;
  __syncthreads();
  if (threadIdx.x == 0) {
    int off = 0, roff = 0, dtot = 0;
    for (int w = 0; w < RF_SCAN_THREADS / 32; ++w) dtot += dsum[w];
    for (int n = 0; n < n_nodes; ++n) {
      node_offsets[n] = off;
      pilots_per_node[n] = carry_t[n];
      node_rep_off[n] = roff;
      off += carry_t[n];
      roff += carry_r[n];
    }
    node_offsets[n_nodes] = off;
    counts[0] = off;
    counts[1] = dtot;
    replica_offsets[off] = roff;
  }
}

// Per token: the in-tile prefix by warp scans, then the outputs.  The pilot rows of one node in a
// tile are consecutive, so the per-node pilot stores are coalesced; the replica lists and
// assign_pilot are staged in shared memory and leave as contiguous runs.  Each thread keeps its
// token's sorted keys in its own padded row and reads a node's run back from there.
// Dynamic shared memory: RF_TILE rows of KM + 1 ints, then the RF_TILE * KM staging ints.
template <int KM>
constexpr int rf_emit_smem() { return (RF_TILE * (KM + 1) + RF_TILE * KM) * 4; }

template <int KM>
__global__ void __launch_bounds__(RF_TILE) rbd_fast_emit_kernel(
    const int32_t* __restrict__ ids, int T, int k, int E, int epd, int epn, int n_nodes,
    const int32_t* __restrict__ tile_tok_base, const int32_t* __restrict__ tile_rep_base,
    const int32_t* __restrict__ node_offsets, const int32_t* __restrict__ node_rep_off, int32_t* __restrict__ pilot_token,
    int32_t* __restrict__ pilot_node, int32_t* __restrict__ pilot_device, int32_t* __restrict__ replica_offsets,
    int32_t* __restrict__ replica_expert, int32_t* __restrict__ assign_pilot, int32_t* err) {
  extern __shared__ int32_t rf_sm[];
  __shared__ int wsum[RF_TILE / 32][RF_NODES];
  __shared__ int node_loc[RF_NODES + 1];   // replicas of earlier nodes in this tile
  __shared__ int tok_base[RF_NODES];       // per node: the tile's first pilot row
  __shared__ int rep_gbase[RF_NODES];      // per node: the tile's first replica row
  int32_t* rows = rf_sm;                   // [RF_TILE][KM + 1]: the tile's ids, then each token's sorted keys
  int32_t* sbuf = rf_sm + RF_TILE * (KM + 1);   // [RF_TILE * KM]: replica lists, then assign_pilot
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long t = static_cast<long long>(blockIdx.x) * RF_TILE + threadIdx.x;
  const bool valid = t < T;
  const long long tb = static_cast<long long>(blockIdx.x) * RF_NODES;
  if (threadIdx.x < n_nodes) {
    tok_base[threadIdx.x] = node_offsets[threadIdx.x] + tile_tok_base[tb + threadIdx.x];
    rep_gbase[threadIdx.x] = node_rep_off[threadIdx.x] + tile_rep_base[tb + threadIdx.x];
  }
  int32_t* row = rows + threadIdx.x * (KM + 1);
  unsigned long long cnt;
  (void)err;   // rbd_fast_count flagged bad ids
  const FastDiv node_of(epn), dev_of(epd);
  {
    int v[KM];
    if (rf_direct<KM>(ids, k)) {
      rf_ids_direct<KM>(ids, t, valid, v);
    } else {
      rf_stage_rows<KM>(ids, T, k, rows);
      rf_ids_row<KM>(row, valid, k, v);
    }
    int key[KM];
    rf_keys<KM>(v, valid, k, E, nullptr, key);
    rf_sort<KM>(key);
#pragma unroll
    for (int s = 0; s < KM; ++s) row[s] = key[s];
    cnt = rf_node_counts<KM>(key, node_of);
  }
  // byte n: the token's replicas on nodes before n = the sorted position of node n's run
  const unsigned long long first = cnt * 0x0101010101010101ull - cnt;
  int c[RF_NODES], ex[RF_NODES];
  // in-warp exclusive prefix of the packed counts, per node
#pragma unroll
  for (int n = 0; n < RF_NODES; ++n) {
    c[n] = rf_packed(cnt, n);
    int a = c[n];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, a, o);
      if (lane >= o) a += y;
    }
    ex[n] = a - c[n];
    if (lane == 31) wsum[warp][n] = a;
  }
  __syncthreads();   // wsum complete
  if (warp == 0) {
    // lane n < RF_NODES: column n of wsum -> exclusive prefix over the warps (the packed fields add
    // independently); the node's replica total -> node_loc by a scan over lanes 0 .. RF_NODES - 1
    int tot = 0;
    if (lane < RF_NODES) {
      int run = 0;
      for (int w = 0; w < RF_TILE / 32; ++w) {
        const int x = wsum[w][lane];
        wsum[w][lane] = run;
        run += x;
      }
      tot = run >> 16;
    }
    int x = tot;
#pragma unroll
    for (int o = 1; o < RF_NODES; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane < RF_NODES) node_loc[lane] = x - tot;
    if (lane == RF_NODES - 1) node_loc[RF_NODES] = x;
  }
  __syncthreads();   // node_loc and the warp prefixes ready
  int idx[RF_NODES];
#pragma unroll
  for (int n = 0; n < RF_NODES; ++n) {
    ex[n] += wsum[warp][n];
    idx[n] = 0;
    if (valid && n < n_nodes && (c[n] & 0xffff)) {
      idx[n] = tok_base[n] + (ex[n] & 0xffff);
      pilot_token[idx[n]] = static_cast<int32_t>(t);
      pilot_node[idx[n]] = n;
      pilot_device[idx[n]] = dev_of(row[rf_node_field(first, n)] >> 8);   // the node's lowest id
      replica_offsets[idx[n]] = rep_gbase[n] + (ex[n] >> 16);
    }
  }
  // replica lists: node n's run of sorted keys at this token's slots of the tile's staging
  if (valid) {
#pragma unroll
    for (int n = 0; n < RF_NODES; ++n) {
      const int cn = rf_node_field(cnt, n), f = rf_node_field(first, n);
      const int at = node_loc[n] + (ex[n] >> 16);
      for (int w = 0; w < cn; ++w) sbuf[at + w] = row[f + w] >> 8;
    }
  }
  __syncthreads();
  for (int n = 0; n < n_nodes; ++n) {
    const int cn = node_loc[n + 1] - node_loc[n];
    const long long g0 = rep_gbase[n];
    for (int i = threadIdx.x; i < cn; i += RF_TILE) replica_expert[g0 + i] = sbuf[node_loc[n] + i];
  }
  __syncthreads();
  // assign_pilot: the tile's [tokens][k] block is contiguous; slot j of a key is its low byte
  if (valid) {
#pragma unroll
    for (int n = 0; n < RF_NODES; ++n) {
      const int cn = rf_node_field(cnt, n), f = rf_node_field(first, n);
      for (int w = 0; w < cn; ++w) sbuf[threadIdx.x * k + (row[f + w] & 0xff)] = idx[n];
    }
  }
  __syncthreads();
  const long long a0 = static_cast<long long>(blockIdx.x) * RF_TILE * k;
  const long long a_end = static_cast<long long>(T) * k;
  for (int i = threadIdx.x; i < RF_TILE * k && a0 + i < a_end; i += RF_TILE) assign_pilot[a0 + i] = sbuf[i];
}

// Launch one of the per-token RBD kernels with the smallest lane group that holds k experts.
#define PFMOE_RBD_LAUNCH(NAME, KERNEL, T_, k_, s_, ...)                                                       \
  do {                                                                                                       \
    const int gsz = (k_) <= 8 ? 8 : ((k_) <= 16 ? 16 : 32);                                                  \
    const int grid = rows_grid((static_cast<long long>(T_) * gsz + 31) / 32);                                 \
    if (gsz == 8) PFMOE_LAUNCH(NAME, s_, (KERNEL<8><<<grid, 256, 0, s_>>>(__VA_ARGS__)));                     \
    else if (gsz == 16) PFMOE_LAUNCH(NAME, s_, (KERNEL<16><<<grid, 256, 0, s_>>>(__VA_ARGS__)));              \
    else PFMOE_LAUNCH(NAME, s_, (KERNEL<32><<<grid, 256, 0, s_>>>(__VA_ARGS__)));                             \
  } while (0)

int rows_grid(long long rows, int warps_per_blk = 8) {
  long long b = (rows + warps_per_blk - 1) / warps_per_blk;
  const long long cap = static_cast<long long>(num_sms()) * 16;
  if (b > cap) b = cap;
  return static_cast<int>(b < 1 ? 1 : b);
}

// Chunk counts -> relative bases + key totals/offsets/tiles: one CTA while the chunks are few, else a
// CTA per strip of keys (strip_scan, whose last CTA scans the keys).  key_tot [K] and the ticket
// (zeroed by the histogram launch) serve the many-chunk path.
constexpr int SMALL_CHUNKS = 64;

int sort_scan(const int32_t* counts, int C, int K, int32_t* totals, int32_t* offsets, int32_t* base, int32_t* tiles,
              int tile_rows, int32_t* key_tot, unsigned* ticket, const char* name, cudaStream_t s) {
  if (C <= SMALL_CHUNKS) {
    PFMOE_LAUNCH(name, s,
                 chunk_scan_kernel<<<1, SCAN_THREADS, 0, s>>>(counts, C, K, totals, offsets, base, tiles, tile_rows));
    return PFMOE_OK;
  }
  PFMOE_LAUNCH(name, s, strip_scan_kernel<<<(K + STRIP_KEYS - 1) / STRIP_KEYS, SCAN_THREADS, 0, s>>>(
                            counts, C, K, base, key_tot, ticket, totals, offsets, tiles, tile_rows));
  return PFMOE_OK;
}

// Tiles of the three-launch long scan for n_max elements (the tile sums need 2 * this many ints).
inline long long long_scan_tiles(long long n_max) { return (n_max + SCAN_TILE - 1) / SCAN_TILE; }
constexpr long long LONG_SCAN_MIN = 4LL * SCAN_TILE;   // below this one CTA scans the array

// The staged scatter needs up to ~95 KB of shared memory (K = 4096 keys, three warps): opt in
// once per device.
template <class Sink, int KEY_BITS>
int scatter_smem_attr() {
  return smem_optin(reinterpret_cast<const void*>(&chunk_scatter_kernel<Sink, KEY_BITS>), 227 * 1024,
                    "chunk_scatter");
}

// Histogram + scatter launches of one stable counting sort.
int sort_hist(const int32_t* keys, long long n_max, const int32_t* n_dev, int K, int C, int32_t* counts,
              unsigned* ticket, int32_t* err, const char* name, cudaStream_t s) {
  const int wpb = warps_per_block(K);
  PFMOE_LAUNCH(name, s, (chunk_hist_kernel<<<C, wpb * 32, K * sizeof(int32_t), s>>>(keys, n_max, n_dev, K, C, counts,
                                                                                   ticket, err)));
  return PFMOE_OK;
}

template <class Sink, int KEY_BITS>
int sort_scatter_as(const int32_t* keys, long long n_max, const int32_t* n_dev, int K, int C, const int32_t* base,
                    const int32_t* key_offsets, const Sink& sink, const char* name, cudaStream_t s) {
  const int wpb = warps_per_block(K);
  PFMOE_TRY((scatter_smem_attr<Sink, KEY_BITS>()));
  PFMOE_LAUNCH(name, s, (chunk_scatter_kernel<Sink, KEY_BITS><<<C, wpb * 32, scatter_smem_bytes(wpb, K), s>>>(
                            keys, n_max, n_dev, K, C, base, key_offsets, sink)));
  return PFMOE_OK;
}

// Equal keys found by ballots over their bits up to 1024 keys, else by __match_any_sync.
template <class Sink>
int sort_scatter(const int32_t* keys, long long n_max, const int32_t* n_dev, int K, int C, const int32_t* base,
                 const int32_t* key_offsets, const Sink& sink, const char* name, cudaStream_t s) {
  if (K <= 256) return sort_scatter_as<Sink, 8>(keys, n_max, n_dev, K, C, base, key_offsets, sink, name, s);
  if (K <= 1024) return sort_scatter_as<Sink, 10>(keys, n_max, n_dev, K, C, base, key_offsets, sink, name, s);
  return sort_scatter_as<Sink, 0>(keys, n_max, n_dev, K, C, base, key_offsets, sink, name, s);
}

template <int KM>
static int rbd_fast_launch(const int32_t* ids, int T, int k, int E, int epd, int epn, int n_nodes, int32_t* ppn,
                           int32_t* noff, int32_t* ptok, int32_t* pnode, int32_t* pdev, int32_t* roff, int32_t* rexp,
                           int32_t* ap, int32_t* counts, int32_t* tile_cnt, int32_t* tile_rep, int32_t* tile_dev,
                           int32_t* node_rep_off, int32_t* err, cudaStream_t s) {
  const int ntiles = (T + RF_TILE - 1) / RF_TILE;
  if (ntiles > 0)
    PFMOE_LAUNCH("rbd_count", s,
                 (rbd_fast_count_kernel<KM><<<ntiles, RF_TILE, 0, s>>>(ids, T, k, E, epd, epn, tile_cnt, tile_dev,
                                                                      err)));
  PFMOE_TRY(smem_optin(reinterpret_cast<const void*>(&rbd_fast_scan_kernel), RF_SCAN_SMEM, "rbd_scan_nodes"));
  PFMOE_LAUNCH("rbd_scan_nodes", s,
               (rbd_fast_scan_kernel<<<1, RF_SCAN_THREADS, RF_SCAN_SMEM, s>>>(ntiles, n_nodes, tile_cnt, tile_rep,
                                                                              tile_dev, ppn, noff, node_rep_off,
                                                                              counts, roff)));
  PFMOE_TRY(smem_optin(reinterpret_cast<const void*>(&rbd_fast_emit_kernel<KM>), rf_emit_smem<KM>(), "rbd_emit"));
  if (ntiles > 0)
    PFMOE_LAUNCH("rbd_emit", s,
               (rbd_fast_emit_kernel<KM><<<ntiles, RF_TILE, rf_emit_smem<KM>(), s>>>(ids, T, k, E, epd, epn, n_nodes, tile_cnt, tile_rep,
                                                                    noff, node_rep_off, ptok, pnode, pdev, roff, rexp,
                                                                    ap, err)));
  return PFMOE_OK;
}

static int rbd_fast_impl(const int32_t* ids, int T, int k, int E, int epd, int epn, int n_nodes, int32_t* ppn,
                         int32_t* noff, int32_t* ptok, int32_t* pnode, int32_t* pdev, int32_t* roff, int32_t* rexp,
                         int32_t* ap, int32_t* counts, void* ws, int32_t* err, cudaStream_t s) {
  const size_t tiles = (static_cast<size_t>(T) + RF_TILE - 1) / RF_TILE;
  int32_t* tile_cnt = static_cast<int32_t*>(ws);
  int32_t* tile_rep = tile_cnt + tiles * RF_NODES;
  int32_t* tile_dev = tile_rep + tiles * RF_NODES;
  int32_t* node_rep_off = tile_dev + tiles;
  if (k <= 8)
    return rbd_fast_launch<8>(ids, T, k, E, epd, epn, n_nodes, ppn, noff, ptok, pnode, pdev, roff, rexp, ap, counts,
                              tile_cnt, tile_rep, tile_dev, node_rep_off, err, s);
  if (k <= 16)
    return rbd_fast_launch<16>(ids, T, k, E, epd, epn, n_nodes, ppn, noff, ptok, pnode, pdev, roff, rexp, ap, counts,
                               tile_cnt, tile_rep, tile_dev, node_rep_off, err, s);
  return rbd_fast_launch<32>(ids, T, k, E, epd, epn, n_nodes, ppn, noff, ptok, pnode, pdev, roff, rexp, ap, counts,
                             tile_cnt, tile_rep, tile_dev, node_rep_off, err, s);
}

}  // namespace

// Counts and bases ([C][K] each), key totals [K], the strip scan's ticket.
size_t csort_ws_bytes(long long n_max, int K) {
  const long long C = (n_max + chunk_keys(K) - 1) / chunk_keys(K);
  return static_cast<size_t>(2 * (C > 0 ? C : 1) * static_cast<long long>(K) + K + 1) * sizeof(int32_t);
}

int pft_build_impl(const int32_t* ids, const float* w, int T, int E, int k, int32_t* tpe, int32_t* offsets,
                   int32_t* token_ids, int32_t* expert_ids, float* cw, int32_t* pos, int32_t* tile_offsets,
                   void* ws, int32_t* err, cudaStream_t s) {
  const long long N = static_cast<long long>(T) * k;
  const int C = static_cast<int>((N + chunk_keys(E) - 1) / chunk_keys(E));
  int32_t* counts = static_cast<int32_t*>(ws);
  int32_t* base = counts + static_cast<long long>(C) * E;
  int32_t* key_tot = base + static_cast<long long>(C) * E;
  unsigned* ticket = reinterpret_cast<unsigned*>(key_tot + E);
  if (C > 0) PFMOE_TRY(sort_hist(ids, N, nullptr, E, C, counts, ticket, err, "pft_hist", s));
  PFMOE_TRY(sort_scan(counts, C, E, tpe, offsets, base, tile_offsets, 128, key_tot, ticket, "pft_scan", s));
  PftSink sink{w, k, k > 1 ? ~0ull / static_cast<unsigned>(k) + 1 : 0ull, pos, token_ids, expert_ids, cw};
  if (C > 0) PFMOE_TRY(sort_scatter<PftSink>(ids, N, nullptr, E, C, base, offsets, sink, "pft_scatter", s));
  return PFMOE_OK;
}

// Workspace of the plan for maps of at most RF_NODES nodes: two [tiles][RF_NODES] arrays, one [tiles].
static size_t rbd_fast_ws_bytes(int T) {
  const size_t tiles = (static_cast<size_t>(T) + RF_TILE - 1) / RF_TILE;
  return (2 * tiles * RF_NODES + tiles + 64) * sizeof(int32_t);
}

// The plan without a sort serves maps of at most RF_NODES nodes whose ids fit the 16-bit fast division
// and the id * 256 + slot sort keys.
static bool rbd_fast_ok(int E, int n_nodes) { return n_nodes <= RF_NODES && E <= (1 << 16); }

size_t rbd_ws_bytes(int T, int k, int E, int n_nodes) {
  if (rbd_fast_ok(E, n_nodes)) return rbd_fast_ws_bytes(T);
  const long long pmax = static_cast<long long>(T) * (k < n_nodes ? k : n_nodes);
  const long long lt = long_scan_tiles(pmax > T ? pmax : T);
  const size_t ints = 3 * static_cast<size_t>(T) + 5 * static_cast<size_t>(pmax) + 2 * static_cast<size_t>(lt) + 128;
  return ints * sizeof(int32_t) + csort_ws_bytes(pmax, n_nodes) + 256;
}

int rbd_plan_impl(const int32_t* ids, int T, int k, int E, int epd, int dpn, int32_t* pilots_per_node,
                  int32_t* node_offsets, int32_t* pilot_token, int32_t* pilot_node, int32_t* pilot_device,
                  int32_t* replica_offsets, int32_t* replica_expert, int32_t* assign_pilot, int32_t* counts,
                  void* ws, int32_t* err, cudaStream_t s) {
  const int epn = epd * dpn;
  const int n_nodes = E / epn;
  if (rbd_fast_ok(E, n_nodes)) return rbd_fast_impl(ids, T, k, E, epd, epn, n_nodes, pilots_per_node, node_offsets,
                                                pilot_token, pilot_node, pilot_device, replica_offsets, replica_expert,
                                                assign_pilot, counts, ws, err, s);
  const long long pmax = static_cast<long long>(T) * (k < n_nodes ? k : n_nodes);
  int32_t* p = static_cast<int32_t*>(ws);
  int32_t* ucount = p; p += T;
  int32_t* dcount = p; p += T;
  int32_t* pbase = p; p += T;
  int32_t* pkey = p; p += pmax;
  int32_t* ptoken = p; p += pmax;
  int32_t* prc = p; p += pmax;
  int32_t* psorted = p; p += pmax;
  int32_t* rc_sorted = p; p += pmax;
  const long long lt = long_scan_tiles(pmax > T ? pmax : T);
  int32_t* tsum_a = p; p += lt;
  int32_t* tsum_b = p; p += lt;
  p += 64 - ((p - static_cast<int32_t*>(ws)) & 63);   // keep 256-byte alignment
  const int C = static_cast<int>((pmax + chunk_keys(n_nodes) - 1) / chunk_keys(n_nodes));
  int32_t* ccounts = p; p += static_cast<long long>(C > 0 ? C : 1) * n_nodes;
  int32_t* cbase = p;

  PFMOE_RBD_LAUNCH("rbd_count", rbd_count_kernel, T, k, s, ids, T, k, E, epd, epn, ucount, dcount, err);
  if (T < LONG_SCAN_MIN) {
    PFMOE_LAUNCH("rbd_scan_tokens", s, rbd_scan_kernel<<<1, SCAN_THREADS, 0, s>>>(ucount, dcount, T, pbase, counts));
  } else {
    const int nt = static_cast<int>(long_scan_tiles(T));
    PFMOE_LAUNCH("rbd_scan_tokens", s,
                 tile_sum_kernel<<<nt, SCAN_THREADS, 0, s>>>(ucount, dcount, T, nullptr, tsum_a, tsum_b));
    PFMOE_LAUNCH("rbd_scan_tokens", s,
                 tile_offsets_kernel<<<1, SCAN_THREADS, 0, s>>>(tsum_a, tsum_b, nt, counts, counts + 1, nullptr, 0,
                                                                nullptr));
    PFMOE_LAUNCH("rbd_scan_tokens", s, tile_scan_kernel<<<nt, SCAN_THREADS, 0, s>>>(ucount, T, nullptr, tsum_a, pbase));
  }
  PFMOE_RBD_LAUNCH("rbd_emit", rbd_emit_kernel, T, k, s, ids, T, k, E, epd, epn, pbase, pkey, ptoken, prc, err);
  int32_t* node_tot = cbase + static_cast<long long>(C > 0 ? C : 1) * n_nodes;
  unsigned* ticket = reinterpret_cast<unsigned*>(node_tot + n_nodes);
  if (C > 0) PFMOE_TRY(sort_hist(pkey, pmax, counts, n_nodes, C, ccounts, ticket, err, "rbd_hist", s));
  PFMOE_TRY(sort_scan(ccounts, C, n_nodes, pilots_per_node, node_offsets, cbase, nullptr, 0, node_tot, ticket,
                      "rbd_scan_nodes", s));
  if (C > 0) {
    RbdSink sink{ptoken, prc, pilot_token, pilot_node, rc_sorted, psorted};
    PFMOE_TRY(sort_scatter<RbdSink>(pkey, pmax, counts, n_nodes, C, cbase, node_offsets, sink, "rbd_scatter", s));
  }
  if (pmax < LONG_SCAN_MIN) {
    PFMOE_LAUNCH("rbd_scan_replicas", s,
                 excl_scan_kernel<<<1, SCAN_THREADS, 0, s>>>(rc_sorted, pmax, counts, replica_offsets));
  } else {
    // P = counts[0] lives on the device: tiles past it sum to zero and write nothing
    const int nt = static_cast<int>(long_scan_tiles(pmax));
    PFMOE_LAUNCH("rbd_scan_replicas", s,
                 tile_sum_kernel<<<nt, SCAN_THREADS, 0, s>>>(rc_sorted, nullptr, pmax, counts, tsum_a, nullptr));
    PFMOE_LAUNCH("rbd_scan_replicas", s,
                 tile_offsets_kernel<<<1, SCAN_THREADS, 0, s>>>(tsum_a, nullptr, nt, nullptr, nullptr, replica_offsets,
                                                                pmax, counts));
    PFMOE_LAUNCH("rbd_scan_replicas", s,
                 tile_scan_kernel<<<nt, SCAN_THREADS, 0, s>>>(rc_sorted, pmax, counts, tsum_a, replica_offsets));
  }
  PFMOE_RBD_LAUNCH("rbd_final", rbd_final_kernel, T, k, s, ids, T, k, E, epd, epn, pbase, psorted, replica_offsets,
                   assign_pilot, replica_expert, pilot_device, err);
  return PFMOE_OK;
}

}  // namespace pfmoe
