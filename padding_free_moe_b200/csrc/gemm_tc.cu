// Persistent GEMMs on the 5th-generation tensor cores (sm_100a):
// TMA -> shared-memory ring -> tcgen05.mma (one issuing thread) -> TMEM
// accumulators (double-buffered) -> epilogue warps.  BF16 operands, FP32
// accumulation.  Two kernels cover every contraction of the padding-free layer:
//
// grouped_gemm_tn_kernel (two-SM, cta_group::2) -- the row-grouped expert GEMMs
//   (H1/H3/A = SwiGLU(X W1, X W3), O = A W2, dA = dO W2^T, dX = dH1 W1^T + dH3 W3^T).
//   The PFT rows of expert g are the segment [seg[g], seg[g+1]) (X-MoE article
//   §2.1.2: one GEMM per expert over its unpadded rows).  The expert's weights
//   are the MMA's A operand (256 output features per CTA pair) and its tokens the
//   B operand (N = the tile's token count rounded up to 32), and the epilogue
//   transposes back to [token, feature] rows.
//
// grouped_gemm_kernel (one-SM) in two modes:
//   KG (K-grouped): the reduction runs over a segment (weight gradients
//      dW_g = X_g^T dH_g, and the gate's dWg split along T); each group writes its
//      own [M, N] output.  K rows past the segment end are zeroed in shared memory
//      by a dedicated warp before the MMA reads the block.
//   RG (row-grouped, dense): the gate logits X Wg, split along K when the output
//      has too few tiles to fill the GPU.
//
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer (and TMEM allocator),
// warps 2..5 = epilogue (TMEM lane quarter q = warp % 4), warp 6 (K-grouped
// launches only) = K-tail zeroing.  Every wait on an mbarrier is bounded
// (%globaltimer); on expiry the kernel sets PFMOE_DEV_TIMEOUT, drains its own
// copies and MMAs, frees TMEM and returns.  The token-as-N epilogue warps also
// meet at a named barrier once or twice per 32-token chunk; all four take the
// same barrier steps and leave their tile loop together through a barrier vote,
// so none waits at a barrier that another has left.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace pfmoe {
namespace tc {

constexpr int BM = 128;          // MMA M (one CTA)
constexpr int BK = 64;           // K elements per stage (one 128-byte swizzle row of BF16)
constexpr int MAX_STAGES = 8;
constexpr int THREADS = 192;
// Token-as-N kernel with the token rows gathered into the B ring (no PFT copy of x): four more
// warps copy the rows with 16-byte cp.async (TMA tile::gather4 moves 512 bytes per copy and
// measured 16 GB/s per SM on this part, against 83 GB/s for four warps of cp.async).
constexpr int GATHER_WARPS = 4;
constexpr int THREADS_GATHER = THREADS + 32 * (GATHER_WARPS + 1);   // + one relay warp
// K-grouped (weight-gradient) launches: KG_EPI_WARPS epilogue warps (a multiple of 4; with 8, two
// per TMEM lane quarter each write half of a tile's column blocks) and a K-tail zeroing warp after
// them.  Four warps with two staging slabs each measured as fast as eight with one or two.
constexpr int KG_EPI_WARPS = 4;
constexpr int KG_STAGE_BUFS = 2;         // staging slabs per KG epilogue warp
constexpr int KG_ZERO_WARP = 2 + KG_EPI_WARPS;
constexpr int THREADS_KG = (KG_ZERO_WARP + 1) * 32;
constexpr int BOX_BYTES = 64 * 128;      // one 64 x 64 BF16 box (MN-major block)
constexpr int A_BYTES = BM * BK * 2;     // 16 KB

constexpr unsigned long long kTimeoutNs = 2000000000ull;

enum Mode { RG = 0, KG = 1 };
// K depth of one ring stage of the one-SM kernel (template argument KBK): 128 where three or more
// stages still fit (gate dWg: bn = 64), which doubles the operand copies and halves the MMA
// issuer's barrier handshakes; 64 for the 256-wide expert weight-gradient tiles, where a
// 128-deep stage leaves room for only two stages and measured slower.
constexpr int KG_BK = 2 * BK;
enum Epi { EPI_STORE_BF16 = 0, EPI_STORE_F32 = 1, EPI_SWIGLU_FWD = 2, EPI_SWIGLU_BWD = 3, EPI_SPLIT_BF16 = 4,
           EPI_REDADD_BF16 = 5 };   // REDADD: D += acc (BF16), full slabs by TMA reduce-add

struct Params {
  CUtensorMap tmA[2];
  CUtensorMap tmB[2];
  CUtensorMap tmD[3];  // output maps for TMA stores from the staged epilogue (box 128 B x 32 rows)
  int tma_store;       // 1: tmD[] are valid
  int mode;
  int b_major;       // RG: 0 = K-major B (weights [G, N, K]), 1 = MN-major B (weights [G, K, N]); KG: 1
  int a_major;       // token-as-N kernel: 0 = K-major weights [G, F, K], 1 = MN-major weights [G, K, F]
  int a_merged;      // MN-major A map is the 4-D block view (one copy fetches every 64-wide block of a stage)
  int b_merged;      // same for the MN-major B maps
  int fstep;         // token-as-N kernel: output features per pair tile (256, or 128 with nsplit)
  int tn_nb;         // token-as-N kernel: epilogue chunk buffers (2; 1 where shared memory is short)
  int bn;            // MMA N: multiple of 64, <= 256
  int nsplit;        // 1: B tile columns [0, bn/2) come from tmB[0], [bn/2, bn) from tmB[1]
  int M;             // KG: rows of each group's output
  int Nout;          // output columns
  int k0_blocks;     // RG: 64-wide K blocks read from source 0
  int k1_blocks;     // RG: then from source 1 (K split; 0 = none)
  const int* seg;    // [G+1] segment offsets, or null for one dense segment [0, dense_len)
  const int* tiles;  // RG: [G+1] prefix of 128-row M tiles per group (null when dense)
  int G;
  int dense_len;
  int stages;
  int ksplit;        // dense problems only: K is cut into ksplit parts, part s writes output slice s
  int kchunk;        // KG dense: K rows per part (multiple of KG_BK)
  void* D0;
  void* D1;
  void* D2;
  const void* X0;    // SWIGLU_BWD: H1
  const void* X1;    // SWIGLU_BWD: H3
  const float* bias; // STORE_F32: optional per-column bias
  long long ldd;     // output row stride (elements)
  long long d_gstride;  // KG: elements between consecutive groups' outputs
  const int32_t* gather_ids;  // token-as-N with gathered B: PFT row -> token (token_ids)
  const void* gather_src;      // token rows [T, gather_ld] the B operand is gathered from
  long long gather_ld;
  int32_t* err;
};

struct Tile {
  int g;
  int row0;    // RG: first PFT row; KG: first output row (M)
  int rows;    // valid rows (<= 128)
  int n0;      // first output column
  int nk;      // K blocks
  int krow0;   // KG: first K row of the segment
  int kvalid;  // KG: valid K rows in the last block
  int kb0;     // RG: first K block (split-K)
  int split;   // RG: split-K part (output slice)
};

// ------------------------------------------------------------------ PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ uint32_t mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok;
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait.  Returns false if the wait expired or another role aborted.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int32_t* err, bool honour_abort = true,
                                         unsigned long long limit_ns = kTimeoutNs) {
  for (int i = 0; i < 128; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (honour_abort && *abort_flag) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort_flag = 1;
      dev_error(err, PFMOE_DEV_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* tm, uint32_t bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// 4-D form for the block view of an MN-major tensor: coordinates (0, k, block, group).
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* tm, uint32_t bar, int c0, int c1, int c2,
                                            int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* tm) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_mma(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns: thread i gets lane (base lane + i).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 format: version 1 at bit 46,
// layout type 2 = SWIZZLE_128B at bits 61..63; addresses and offsets in 16-byte units).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor for kind::f16: D=F32, A=B=BF16, dense, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// ----------------------------------------------------------------- tile schedule
__device__ __forceinline__ int n_step(const Params& p) { return p.nsplit ? p.bn / 2 : p.bn; }

template <int MODE>
__device__ __forceinline__ int total_tiles(const Params& p) {
  const int ns = n_step(p);
  const int NT = (p.Nout + ns - 1) / ns;
  if constexpr (MODE == RG) return (p.dense_len + BM - 1) / BM * p.ksplit * NT;
  return p.G * ((p.M + BM - 1) / BM) * NT;
}

template <int MODE, int KBK>
__device__ __forceinline__ Tile decode(const Params& p, int t) {
  Tile tl;
  const int ns = n_step(p);
  const int NT = (p.Nout + ns - 1) / ns;
  if constexpr (MODE == RG) {
    // dense rows [0, dense_len), optionally split along K into ksplit output slices
    const int mtg = (p.dense_len + BM - 1) / BM;
    const int split = t / (mtg * NT);
    const int local = t - split * mtg * NT;
    const int n_idx = local / mtg;
    const int m_loc = local - n_idx * mtg;
    tl.g = 0;
    tl.row0 = m_loc * BM;
    tl.rows = min(BM, p.dense_len - tl.row0);
    tl.n0 = n_idx * ns;
    const int nk_all = p.k0_blocks + p.k1_blocks;
    const int kbs = (nk_all + p.ksplit - 1) / p.ksplit;
    tl.split = split;
    tl.kb0 = split * kbs;
    tl.nk = max(0, min(kbs, nk_all - tl.kb0));
    tl.krow0 = 0;
    tl.kvalid = BK;
  } else {
    const int MT = (p.M + BM - 1) / BM;
    const int per = MT * NT;
    const int g = t / per;
    const int rem = t - g * per;
    const int n_idx = rem / MT;
    const int m_idx = rem - n_idx * MT;
    const int s0 = p.seg ? p.seg[g] : g * p.kchunk;
    const int s1 = p.seg ? p.seg[g + 1] : min(p.dense_len, s0 + p.kchunk);
    const int len = max(0, s1 - s0);
    tl.split = 0;
    tl.kb0 = 0;
    tl.g = g;
    tl.row0 = m_idx * BM;
    tl.rows = min(BM, p.M - tl.row0);
    tl.n0 = n_idx * ns;
    tl.nk = (len + KBK - 1) / KBK;
    tl.krow0 = s0;
    tl.kvalid = len - (tl.nk - 1) * KBK;
  }
  return tl;
}

// Sigmoid for the BF16 epilogues: fast exponential and division (relative error ~1e-6,
// far below the 2^-9 rounding of the BF16 results they feed).
__device__ __forceinline__ float sigmoid_fast(float u) { return __fdividef(1.0f, 1.0f + __expf(-u)); }

// ------------------------------------------------------------- direct epilogue
// Row-grouped (dense gate) tiles: each thread stores its own FP32 row straight from
// registers (16-byte vectors); the tiles are few and their K loops long.
template <typename T>
__device__ __forceinline__ void store_row_chunk(T* dst, const float* v, int ncols_valid) {
  // Store up to 32 values of one row; ncols_valid is a multiple of 8 (BF16) or 4 (F32) or >= 32.
  constexpr int VN = Vec<T>::n;
#pragma unroll
  for (int i = 0; i < 32; i += VN)
    if (i < ncols_valid) store16<T>(dst + i, v + i);
}

template <int EPI>
__device__ __forceinline__ void epilogue_tile_direct(const Params& p, const Tile& tl, uint32_t tacc, int r) {
  const bool row_ok = r < tl.rows;
  const long long grow = static_cast<long long>(tl.row0) + r;
  const bool zero = tl.nk == 0;
  if constexpr (EPI == EPI_STORE_BF16 || EPI == EPI_STORE_F32) {
    using T = typename std::conditional<EPI == EPI_STORE_F32, float, __nv_bfloat16>::type;
    T* D = static_cast<T*>(p.D0) + (p.mode == KG ? tl.g : tl.split) * p.d_gstride;
    for (int c = 0; c < p.bn; c += 32) {
      const int col = tl.n0 + c;
      if (col >= p.Nout) break;
      float v[32];
      if (!zero) tmem_ld32(tacc + c, v);
      else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      if (EPI == EPI_STORE_F32 && p.bias) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (col + i < p.Nout) v[i] += p.bias[col + i];
      }
      if (row_ok) store_row_chunk<T>(D + grow * p.ldd + col, v, p.Nout - col);
    }
  }
}

// -------------------------------------------------------- staged epilogue
// Each epilogue warp owns a 32-row slab of the 128-row accumulator (its TMEM lane
// quarter).  Values leave TMEM one row per thread; they are written to a per-warp
// 32 x 128-byte staging buffer in shared memory (16-byte chunks swizzled by row so
// both the row-wise writes and the column-wise reads are bank-conflict free) and
// copied to global memory four rows per instruction, eight lanes per 128-byte row
// segment.  Every global store is then part of a full 128-byte line.  Used for
// K-grouped (weight-gradient) tiles, whose short K loops leave the epilogue exposed.
constexpr int STAGE_BYTES_PER_WARP = 32 * 128;   // one 32-row x 128-byte slab

__device__ __forceinline__ void tmem_ld32_async(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// 64 consecutive accumulator columns of this thread's row (two loads, one wait).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  uint32_t r[64];
  tmem_ld32_async(taddr, r);
  tmem_ld32_async(taddr + 32, r + 32);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint32_t stg_addr(uint32_t stg, int row, int chunk) {
  return stg + row * 128 + ((chunk ^ (row & 7)) << 4);
}
__device__ __forceinline__ void st_shared16(uint32_t addr, uint4 u) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(u.x), "r"(u.y), "r"(u.z), "r"(u.w)
               : "memory");
}
__device__ __forceinline__ uint4 ld_shared16(uint32_t addr) {
  uint4 u;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "r"(addr)
               : "memory");
  return u;
}

// Thread `lane` writes row `lane` of the slab: 64 BF16 values (or 32 FP32 values) = 128 bytes.
template <typename T>
__device__ __forceinline__ void stage_row(uint32_t stg, int lane, const float* v) {
  constexpr int VN = Vec<T>::n;
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    uint4 u;
    if constexpr (sizeof(T) == 4) {
      u.x = __float_as_uint(v[4 * c]); u.y = __float_as_uint(v[4 * c + 1]);
      u.z = __float_as_uint(v[4 * c + 2]); u.w = __float_as_uint(v[4 * c + 3]);
    } else {
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
      for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[VN * c + 2 * i], v[VN * c + 2 * i + 1]);
    }
    st_shared16(stg_addr(stg, lane, c), u);
  }
}

// Staged slab -> global rows base + row * stride (bytes); rows >= rows_valid and bytes >= bytes_valid are skipped.
__device__ __forceinline__ void copy_out(uint32_t stg, int lane, char* base, long long stride, int rows_valid,
                                         int bytes_valid) {
  const int chunk = lane & 7;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int row = it * 4 + (lane >> 3);
    const uint4 u = ld_shared16(stg_addr(stg, row, chunk));
    if (row < rows_valid && chunk * 16 < bytes_valid)
      *reinterpret_cast<uint4*>(base + row * stride + chunk * 16) = u;
  }
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* tm, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
// Element-wise add of the staged box into global memory (the reduction runs in L2; one add per element).
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* tm, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tm)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

// Staged BF16 slab added to global rows (read, add in float32, round, write); rows >= rows_valid and
// bytes >= bytes_valid are skipped.  Every element has one owner, so there is no race.
__device__ __forceinline__ void copy_out_add_bf16(uint32_t stg, int lane, char* base, long long stride, int rows_valid,
                                                  int bytes_valid) {
  const int chunk = lane & 7;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int row = it * 4 + (lane >> 3);
    const uint4 u = ld_shared16(stg_addr(stg, row, chunk));
    if (row < rows_valid && chunk * 16 < bytes_valid) {
      uint4* g = reinterpret_cast<uint4*>(base + row * stride + chunk * 16);
      uint4 o = *g;
      const __nv_bfloat162* a = reinterpret_cast<const __nv_bfloat162*>(&u);
      __nv_bfloat162* b = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 fa = __bfloat1622float2(a[i]), fb = __bfloat1622float2(b[i]);
        b[i] = __floats2bfloat162_rn(fa.x + fb.x, fa.y + fb.y);
      }
      *g = o;
    }
  }
}

// Per-warp staging state: KG_STAGE_BUFS 4 KB slabs used in turn.
struct Stager {
  uint32_t base;
  int seq;
};

// Stage one 32-row x 128-byte slab and write it out: a full slab goes out as one TMA store
// (the staging layout is the TMA 128-byte swizzle; the store clips at the tensor bounds);
// a slab with missing rows goes out with masked vector stores.  One bulk group is committed
// per slab, so "at most KG_STAGE_BUFS - 1 groups pending" means the slab about to be reused is free.
template <typename T, bool ADD = false>
__device__ __forceinline__ void emit(Stager& st, int lane, const float* v, const CUtensorMap* tm, int c0, int c1,
                                     int c2, T* dst_row0, long long ldd, int rows_valid, int cols_valid) {
  const uint32_t buf = st.base + (st.seq % KG_STAGE_BUFS) * STAGE_BYTES_PER_WARP;
  ++st.seq;
  // the slab about to be written was last read by the store KG_STAGE_BUFS groups ago
  if (lane == 0) asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(KG_STAGE_BUFS - 1) : "memory");
  __syncwarp();
  stage_row<T>(buf, lane, v);
  if (tm && rows_valid == 32) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) {
      if constexpr (ADD) tma_reduce_add_3d(tm, buf, c0, c1, c2);
      else tma_store_3d(tm, buf, c0, c1, c2);
    }
  } else {
    __syncwarp();
    if constexpr (ADD)
      copy_out_add_bf16(buf, lane, reinterpret_cast<char*>(dst_row0), ldd * static_cast<long long>(sizeof(T)),
                        rows_valid, min(128, cols_valid * static_cast<int>(sizeof(T))));
    else
      copy_out(buf, lane, reinterpret_cast<char*>(dst_row0), ldd * static_cast<long long>(sizeof(T)), rows_valid,
               min(128, cols_valid * static_cast<int>(sizeof(T))));
  }
  if (lane == 0) asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until every TMA store this warp issued has written global memory.
__device__ __forceinline__ void emit_drain(int lane) {
  if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  __syncwarp();
}

__device__ __forceinline__ const CUtensorMap* tmd(const Params& p, int i) {
  return p.tma_store ? &p.tmD[i] : nullptr;
}

// Warp (q, half) of nhalves warps per lane quarter writes the 64-column blocks b (32-column chunks
// for FP32) with b % nhalves == half.
template <int EPI>
__device__ __forceinline__ void epilogue_tile(const Params& p, const Tile& tl, uint32_t tacc, int q, int lane,
                                              Stager& stg, int half, int nhalves) {
  const int slab0 = q * 32;
  const int rows_valid = max(0, min(32, tl.rows - slab0));
  const long long grow0 = static_cast<long long>(tl.row0) + slab0;
  const bool zero = tl.nk == 0;
  const int tz = p.mode == KG ? tl.g : 0;   // third output coordinate: expert / split part
  if constexpr (EPI == EPI_STORE_BF16 || EPI == EPI_SPLIT_BF16 || EPI == EPI_REDADD_BF16) {
    const int nparts = EPI == EPI_SPLIT_BF16 ? 2 : 1;
    const int width = EPI == EPI_SPLIT_BF16 ? p.bn / 2 : p.bn;
    const long long goff = p.mode == KG ? tl.g * p.d_gstride : 0;
    for (int part = 0; part < nparts; ++part) {
      __nv_bfloat16* D = static_cast<__nv_bfloat16*>(part == 0 ? p.D0 : p.D1) + goff;
      for (int c = 0; c < width; c += 64) {
        const int col = tl.n0 + c;
        if (col >= p.Nout) break;
        if (((part * width + c) / 64) % nhalves != half) continue;
        float v[64];
        if (!zero) tmem_ld64(tacc + part * width + c, v);
        else {
#pragma unroll
          for (int i = 0; i < 64; ++i) v[i] = 0.f;
        }
        emit<__nv_bfloat16, EPI == EPI_REDADD_BF16>(stg, lane, v, tmd(p, part), col, static_cast<int>(grow0), tz,
                                                   D + grow0 * p.ldd + col, p.ldd, rows_valid, p.Nout - col);
      }
    }
  } else if constexpr (EPI == EPI_STORE_F32) {
    float* D = static_cast<float*>(p.D0) + (p.mode == KG ? tl.g * p.d_gstride : 0);
    for (int c = 0; c < p.bn; c += 32) {
      const int col = tl.n0 + c;
      if (col >= p.Nout) break;
      if ((c / 32) % nhalves != half) continue;
      float v[32];
      if (!zero) {
        uint32_t r[32];
        tmem_ld32_async(tacc + c, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      if (p.bias) {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (col + i < p.Nout) v[i] += p.bias[col + i];
      }
      emit(stg, lane, v, tmd(p, 0), col, static_cast<int>(grow0), tz, D + grow0 * p.ldd + col, p.ldd, rows_valid,
           p.Nout - col);
    }
  }
}

// ---------------------------------------------------------------------- kernel
template <int EPI, int MODE, int KBK>
__global__ void __launch_bounds__(MODE == KG ? THREADS_KG : THREADS, 1) grouped_gemm_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  constexpr uint32_t a_bytes = BM * KBK * 2;
  constexpr uint32_t blk = KBK * 128;        // one MN-major block: 64 columns x KBK K rows
  const uint32_t b_bytes = static_cast<uint32_t>(p.bn) * KBK * 2;
  const uint32_t stage_bytes = a_bytes + b_bytes;
  uint8_t* stage_area = smem + S * stage_bytes;                       // epilogue staging (K-grouped only)
  constexpr bool STAGED = MODE == KG || EPI == EPI_REDADD_BF16;   // staged epilogue (slabs + TMA stores)
  uint8_t* bar_area = stage_area + (STAGED ? KG_EPI_WARPS * KG_STAGE_BUFS * STAGE_BYTES_PER_WARP : 0);
  uint64_t* full = reinterpret_cast<uint64_t*>(bar_area);
  uint64_t* empty = full + MAX_STAGES;
  uint64_t* acc_full = empty + MAX_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* ready = drain + 1;   // K-grouped: stage s landed and its segment-tail rows are zero
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ready + MAX_STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t tmem_cols = p.bn * 2 <= 128 ? 128 : (p.bn * 2 <= 256 ? 256 : 512);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), (MODE == KG ? KG_EPI_WARPS : 4) * 32);
    }
    mbar_init(smem_u32(drain), 1);
    for (int z = 0; z < MAX_STAGES; ++z) mbar_init(smem_u32(&ready[z]), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&p.tmA[0]);
    prefetch_tmap(&p.tmB[0]);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int ntiles = total_tiles<MODE>(p);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Two issuing lanes (per-SM TMA delivery rises a few percent with two issuers): lane 0 posts
    // the stage's byte count and loads A, lane 1 loads B.  The stage's phase completes only after
    // lane 0's arrival and all bytes, so the order of the two lanes' copies does not matter.
    if (lane < 2) {
      uint32_t pending = 0;        // stages with an issued load
      uint32_t pend_parity = 0;    // parity of that load's phase
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const Tile tl = decode<MODE, KBK>(p, t);
        for (int kb = 0; kb < tl.nk; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!wait_bar(smem_u32(&empty[s]), ph ^ 1, abort_flag, p.err)) { ok = false; break; }
          const uint32_t fb = smem_u32(&full[s]);
          if (lane == 0) mbar_expect_tx(fb, stage_bytes);
          const uint32_t sa = smem_u32(smem + s * stage_bytes);
          const uint32_t sb = sa + a_bytes;
          const int nb = p.bn / 64;
          pending |= 1u << s;
          pend_parity = (pend_parity & ~(1u << s)) | (ph << s);
          if constexpr (MODE == RG) {
            // dense gate GEMMs: A rows K-major; B MN-major ([K, N], 64-column boxes) or K-major
            // ([N, K], one box of bn rows)
            const int kk = (tl.kb0 + kb) * BK;
            if (lane == 0) tma_load_3d(sa, &p.tmA[0], fb, kk, tl.row0, 0);
            else if (!p.b_major) tma_load_3d(sb, &p.tmB[0], fb, kk, tl.n0, 0);
            else for (int j = 0; j < nb; ++j) tma_load_3d(sb + j * BOX_BYTES, &p.tmB[0], fb, tl.n0 + 64 * j, kk, 0);
          } else {
            const int krow = tl.krow0 + kb * KBK;
            if (lane == 0) {
              if (p.a_merged) {
                tma_load_4d(sa, &p.tmA[0], fb, 0, krow, tl.row0 / 64, 0);
              } else {
                tma_load_3d(sa, &p.tmA[0], fb, tl.row0, krow, 0);
                tma_load_3d(sa + blk, &p.tmA[0], fb, tl.row0 + 64, krow, 0);
              }
            } else if (p.b_merged) {
              if (p.nsplit) {
                tma_load_4d(sb, &p.tmB[0], fb, 0, krow, tl.n0 / 64, 0);
                tma_load_4d(sb + (nb / 2) * blk, &p.tmB[1], fb, 0, krow, tl.n0 / 64, 0);
              } else {
                tma_load_4d(sb, &p.tmB[0], fb, 0, krow, tl.n0 / 64, 0);
              }
            } else {
              for (int j = 0; j < nb; ++j) {
                int which = 0, nc = tl.n0 + 64 * j;
                if (p.nsplit) {
                  which = j < nb / 2 ? 0 : 1;
                  nc = tl.n0 + 64 * (j < nb / 2 ? j : j - nb / 2);
                }
                tma_load_3d(sb + j * blk, &p.tmB[which], fb, nc, krow, 0);
              }
            }
          }
        }
      }
      // Drain: wait until every load of this stage ring has landed (both lanes wait the same phases).
      for (int s = 0; s < S; ++s)
        if (pending & (1u << s))
          wait_bar(smem_u32(&full[s]), (pend_parity >> s) & 1, abort_flag, p.err, false);
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issuer
    const int a_mn = MODE == KG ? 1 : 0;
    const int b_mn = MODE == KG ? 1 : p.b_major;
    const uint32_t idesc = idesc_bf16(BM, p.bn, a_mn, b_mn);
    const uint32_t a_lbo = a_mn ? blk : 16, b_lbo = b_mn ? blk : 16;   // MN-major: stride between 64-wide blocks
    const uint32_t a_step = a_mn ? 2048 : 32, b_step = b_mn ? 2048 : 32;
    int it = 0, tcount = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tcount) {
      const Tile tl = decode<MODE, KBK>(p, t);
      const int buf = tcount & 1;
      const uint32_t aph = (tcount >> 1) & 1;
      ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&acc_empty[buf]), aph ^ 1, abort_flag, p.err));
      if (!ok) break;
      tc_fence_after();
      const uint32_t tmem_d = tmem_base + buf * p.bn;
      if (tl.nk == 0) {
        if (lane == 0) mbar_arrive(smem_u32(&acc_full[buf]));
        __syncwarp();
        continue;
      }
      for (int kb = 0; kb < tl.nk; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        int kk_count = KBK / 16;
        // K-grouped: the zeroing warp passes every stage on through ready[s] (one phase per ring
        // round, like full[s]) after clearing a segment's tail rows; MMAs of a segment's last block
        // stop at the 16-row step that holds the segment end.
        if (MODE == KG && kb == tl.nk - 1 && tl.kvalid < KBK) kk_count = ((tl.kvalid + 15) & ~15) / 16;
        ok = __all_sync(0xffffffffu, wait_bar(smem_u32(MODE == KG ? &ready[s] : &full[s]), ph, abort_flag, p.err));
        if (!ok) break;
        const uint32_t sa = smem_u32(smem + s * stage_bytes);
        const uint32_t sb = sa + a_bytes;
        tc_fence_after();
        if (lane == 0) {
          // Unrolled with a predicate: one thread issues these, and a rolled loop over a runtime
          // count measured 2-5 % slower on the weight-gradient kernels at d = 7168.
#pragma unroll
          for (int kk = 0; kk < KBK / 16; ++kk) {
            if (kk < kk_count) {
              const uint64_t ad = sdesc(sa + kk * a_step, a_lbo, 1024);
              const uint64_t bd = sdesc(sb + kk * b_step, b_lbo, 1024);
              tc_mma(tmem_d, ad, bd, idesc, (kb | kk) != 0);
            }
          }
          tc_commit(smem_u32(&empty[s]));
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) tc_commit(smem_u32(&acc_full[buf]));
      __syncwarp();
    }
    // Drain: every MMA this thread issued has completed before TMEM is freed.
    if (lane == 0) {
      tc_commit(smem_u32(drain));
      wait_bar(smem_u32(drain), 0, abort_flag, p.err, false);
    }
    __syncwarp();
  } else if (MODE == KG && warp == KG_ZERO_WARP) {
    // ---------------------------------------------------- K-tail zeroing (K-grouped only)
    // Walks every K block in ring order: waits for it to land (full[s]), clears the rows of a
    // segment's last 16-row step past the segment end in every box (A: 2, B: bn/64), and hands
    // the stage to the MMA warp (ready[s]).  Taking part in every round keeps its parity waits
    // unambiguous: it can be at most one phase ahead on any stage.
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      const Tile tl = decode<MODE, KBK>(p, t);
      for (int kb = 0; kb < tl.nk; ++kb, ++it) {
        const int s = it % S;
        ok = __all_sync(0xffffffffu, wait_bar(smem_u32(&full[s]), (it / S) & 1, abort_flag, p.err));
        if (!ok) break;
        if (kb == tl.nk - 1 && tl.kvalid < KBK) {
          const uint32_t sa = smem_u32(smem + s * stage_bytes);
          const int per_box = (((tl.kvalid + 15) & ~15) - tl.kvalid) * 8;   // 16-byte chunks per box
          const int nbox = 2 + p.bn / 64;
          for (int b = 0; b < nbox; ++b)
            for (int i = lane; i < per_box; i += 32)
              st_shared16(sa + b * blk + tl.kvalid * 128 + i * 16, make_uint4(0, 0, 0, 0));
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&ready[s]));
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;           // TMEM lane quarter this warp may access: rows 32q .. 32q+31
    const int half = (warp - 2) / 4;  // K-grouped: which of the two warps of the quarter
    Stager stg{smem_u32(stage_area + (warp - 2) * KG_STAGE_BUFS * STAGE_BYTES_PER_WARP), 0};
    int tcount = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++tcount) {
      const Tile tl = decode<MODE, KBK>(p, t);
      const int buf = tcount & 1;
      const uint32_t aph = (tcount >> 1) & 1;
      if (!__all_sync(0xffffffffu, wait_bar(smem_u32(&acc_full[buf]), aph, abort_flag, p.err))) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * p.bn;
      if constexpr (STAGED) epilogue_tile<EPI>(p, tl, tacc, q, lane, stg, half, KG_EPI_WARPS / 4);
      else epilogue_tile_direct<EPI>(p, tl, tacc, q * 32 + lane);
      tc_fence_before();
      mbar_arrive(smem_u32(&acc_empty[buf]));
    }
    emit_drain(lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// ------------------------------------------------------------------------ host
static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

static int get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return fail(PFMOE_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  return PFMOE_OK;
}

// 3-D tensor map over a row-major tensor [d2][d1][d0] (BF16 or FP32) with a box of
// b0 x b1 x 1 elements and 128-byte swizzle (b0 * element size must be 128 bytes or less).
static int make_tmap_t(CUtensorMap* m, const void* ptr, bool f32, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                       uint32_t b1, const char* what, bool swizzle = true) {
  PFMOE_TRY(get_encode());
  const uint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * es, d0 * d1 * es};
  cuuint32_t box[3] = {b0, b1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                        const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(PFMOE_ERR_CUDA, std::string("cuTensorMapEncodeTiled failed for ") + what + " (CUresult " +
                                    std::to_string(static_cast<int>(r)) + ")");
  return PFMOE_OK;
}

static int make_tmap(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                     uint32_t b1, const char* what) {
  return make_tmap_t(m, ptr, false, d0, d1, d2, b0, b1, what);
}

// Output map for TMA stores of 32-row slabs: BF16 outputs [d2][rows][cols] in 64-column slabs.
static int make_out_map(CUtensorMap* m, void* ptr, uint64_t cols, uint64_t rows, uint64_t d2, const char* what) {
  return make_tmap_t(m, ptr, false, cols, rows, d2, 64, 32, what);
}

// Block view of an MN-major BF16 tensor [g][k][mn] (mn a multiple of 64): a 4-D map over
// (64, k, mn / 64, g) whose box {64, box_k, nblk, 1} lands in shared memory as nblk
// consecutive 64-wide blocks of box_k 128-byte rows -- the same layout as nblk separate
// {64, box_k} boxes, fetched by one copy.  TMA delivery per copy has a fixed cost, so one
// 16-32 KB copy moves operands markedly faster than two to four 8 KB copies.
static int make_tmap_mn(CUtensorMap* m, const void* ptr, uint64_t mn, uint64_t k, uint64_t g, uint32_t box_k,
                        uint32_t nblk, const char* what) {
  PFMOE_TRY(get_encode());
  cuuint64_t dims[4] = {64, k, mn / 64, g};
  cuuint64_t strides[3] = {mn * 2, 128, k * mn * 2};
  cuuint32_t box[4] = {64, box_k, nblk, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(PFMOE_ERR_CUDA, std::string("cuTensorMapEncodeTiled (block view) failed for ") + what + " (CUresult " +
                                    std::to_string(static_cast<int>(r)) + ")");
  return PFMOE_OK;
}

// Output map for the token-as-N kernel: BF16 [rows][cols], boxes of 32 rows x 64 columns with the
// 128-byte swizzle (one staged epilogue block).
static int make_out_map_tn(CUtensorMap* m, void* ptr, uint64_t cols, uint64_t rows, const char* what) {
  return make_tmap_t(m, ptr, false, cols, rows, 1, 64, 32, what, true);
}

static int round_bn(int n) {
  int bn = ((n + 63) / 64) * 64;
  return bn > 256 ? 256 : bn;
}


constexpr int SMEM_LIMIT = 227 * 1024;
// Alignment slack + barriers (512 B), plus the epilogue staging buffers when the launch uses them (K-grouped).
static int smem_fixed(bool staged) {
  return 1024 + 512 + (staged ? KG_EPI_WARPS * KG_STAGE_BUFS * STAGE_BYTES_PER_WARP : 0);
}

static int stage_size(int bn, int kbk) { return (BM + bn) * kbk * 2; }

static int pick_stages(int bn, bool staged, int kbk) {
  int s = (SMEM_LIMIT - smem_fixed(staged)) / stage_size(bn, kbk);
  return s > MAX_STAGES ? MAX_STAGES : s;
}

static size_t smem_bytes(int bn, int stages, bool staged, int kbk) {
  return smem_fixed(staged) + static_cast<size_t>(stages) * stage_size(bn, kbk);
}

// ============================================================================
// Two-SM (tcgen05 cta_group::2) building blocks.
//
// A cluster of two CTAs on one TPC computes one M = 256 tile with MMAs issued by
// the even CTA: each CTA holds 128 rows of A and half of B's columns in its own
// shared memory, and keeps its 128 accumulator rows in its own TMEM.  Both CTAs'
// TMA loads complete on the even CTA's full[s] barrier; the MMA's commits arrive
// on both CTAs' barriers (multicast commit); both CTAs' epilogues arrive on the
// even CTA's acc_empty[b].
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// 16-byte global -> shared copy (cp.async, L2 only); bytes past src_bytes (0 or 16) are zero-filled.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ uint32_t mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok;
}
__device__ __forceinline__ bool wait_bar2(uint32_t bar, uint32_t parity, volatile int* abort_flag, int32_t* err,
                                          bool honour_abort = true) {
  for (int i = 0; i < 128; ++i)
    if (mbar_try_wait_cluster(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (honour_abort && *abort_flag) return false;
    if (globaltimer() - t0 > kTimeoutNs) {
      *abort_flag = 1;
      dev_error(err, PFMOE_DEV_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* tm, uint32_t bar_cluster, int c0,
                                                 int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const CUtensorMap* tm, uint32_t bar_cluster, int c0,
                                                 int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc2(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish2() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_mma2(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Commit arriving on the barrier at the same offset in both CTAs of the pair.
__device__ __forceinline__ void tc_commit2_both(uint32_t bar) {
  const uint16_t mask = 3;
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
                   bar),
               "h"(mask)
               : "memory");
}

// ============================================================================
// Token-as-N two-SM kernel for row-grouped problems.
//
// The expert's weights are the MMA's A operand and its tokens the B operand:
// D^T[f, t] = sum_k W_g[f, k] X[t, k], so TMEM lanes hold output features and
// TMEM columns hold tokens.  A pair tile is M = 256 weight rows (128 per CTA)
// by N = the tile's token count rounded up to 32 (at most 256; CTA v loads
// token columns [vN/2, (v+1)N/2)).  A ragged expert segment therefore costs at
// most 31 spare MMA columns, where 256-row tiles over tokens compute up to 255
// spare rows; on MoE layers with a few hundred tokens per expert that is a
// quarter of the row-major kernel's tensor work.  The epilogue transposes the
// accumulator through shared memory into [token, feature] rows: the four
// epilogue warps of a CTA fill 32-token x 64-feature blocks together and one
// thread writes each block with a single TMA store (fewer, larger copies: the
// per-copy cost of TMA is shared with the operand loads).
//
// With nsplit (SwiGLU forward) a pair tile covers 128 features: CTA v holds
// rows [64v, 64v + 64) of W1^T in TMEM lanes 0..63 and the same rows of W3^T in
// lanes 64..127.  Warps q and q + 2 stage the H1 and H3 bands of one block
// pair; after a barrier all four warps form the A block element-wise from the
// two staged BF16 blocks, so A = SiLU(H1) * H3 of the values that are stored.
constexpr int TN_TOK = 256;             // tokens per pair tile
// K depth of one ring stage: two 64-element sub-blocks, so each mbarrier handshake feeds eight
// K16 MMAs.  Measured on this part: back-to-back M=256 N=256 pair MMAs take ~130 cycles each, and
// a handshake every four of them costs ~30 % of that rate, one every eight none.
constexpr int TN_BK = 2 * BK;
constexpr int TN_SUB = 128 * BK * 2;    // one 64-deep sub-block of 128 rows (16 KB)
constexpr int TN_STAGE = 4 * TN_SUB;    // A: 2 sub-blocks (or 2 feature blocks), B: 2 sub-blocks
constexpr int TN_BLK = 32 * 128;        // one 32-token x 64-feature BF16 block (128-byte rows)

// Epilogue blocks per 32-token chunk: H1, H3, A (SwiGLU forward); dH1 and dH3, two 64-feature
// halves each (SwiGLU backward); two 64-feature halves (plain store).  nb chunk buffers are used
// in turn.
__host__ __device__ constexpr int tn_blocks(int epi) {
  return epi == EPI_SWIGLU_FWD ? 3 : (epi == EPI_SWIGLU_BWD ? 4 : 2);
}
__host__ __device__ constexpr int tn_staging_bytes(int epi, int nb) { return nb * tn_blocks(epi) * TN_BLK; }

struct TnTile {
  int g, tok0, ntok, nmma, f0, nk;
};

__device__ __forceinline__ int tn_feature_tiles(const Params& p) { return (p.Nout + p.fstep - 1) / p.fstep; }

// Pair tiles: expert g has ceil(n_g / 256) token tiles (prefix in pair_off) per feature tile;
// token tiles are the fastest index, so neighbouring CTAs share the same weight block.
__device__ __forceinline__ TnTile decode_tn(const Params& p, const int* pair_off, int t) {
  const int FT = tn_feature_tiles(p);
  int lo = 0, hi = p.G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pair_off[mid] * FT <= t) lo = mid; else hi = mid - 1;
  }
  TnTile tl;
  const int npg = max(1, pair_off[lo + 1] - pair_off[lo]);   // >= 1 whenever tiles[] matches seg[]
  const int local = t - pair_off[lo] * FT;
  const int fi = local / npg;
  const int j = local - fi * npg;
  tl.g = lo;
  tl.tok0 = p.seg[lo] + j * TN_TOK;
  tl.ntok = max(0, min(TN_TOK, p.seg[lo + 1] - tl.tok0));
  tl.nmma = max(32, (tl.ntok + 31) & ~31);                  // a valid MMA shape even for an empty tile
  tl.f0 = fi * p.fstep;
  tl.nk = p.k0_blocks + p.k1_blocks;
  return tl;
}

// Tile order of one pair (P pairs): wave k holds pair tiles [k P, (k + 1) P) as numbered by
// decode_tn, and pair p takes tile k P + p in even waves and k P + P - 1 - p in odd ones.
// Neighbouring tiles (the full and the ragged token tile of one weight block) thus alternate
// between pairs instead of always landing on pairs of the same parity, and the two token tiles
// of a weight block run at the same time, so the block is read from L2 for the second one.
__device__ __forceinline__ bool tn_next(const Params& p, const int* pair_off, int npairs, int pair, int& wave,
                                        TnTile& tl) {
  const int t = wave * npairs + ((wave & 1) ? npairs - 1 - pair : pair);
  if (t >= pair_off[p.G] * tn_feature_tiles(p)) return false;
  tl = decode_tn(p, pair_off, t);
  ++wave;
  return true;
}

__device__ __forceinline__ void st_shared32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_shared32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

// A staged block is [32 tokens][64 features] BF16 with 128-byte rows; 16-byte chunk c of row t
// sits at chunk position c ^ (t & 7) (the TMA 128-byte swizzle).  Epilogue warp q owns the
// 32-feature band (q & 1) of a block: chunks 4 band .. 4 band + 3.
__device__ __forceinline__ uint32_t blk_addr(uint32_t blk, int t, int chunk) {
  return blk + static_cast<uint32_t>(t * 128 + ((chunk ^ (t & 7)) << 4));
}

// Register block (v[j] = token j of feature `lane` of the band) -> staged block.  Lanes 2i and
// 2i + 1 swap one value so that each shared access is a 32-bit word with features 2i, 2i + 1 of
// one token: the even lane writes token j and the odd lane token j + 4, whose swizzled chunk
// lies in the other half of the banks.
__device__ __forceinline__ void blk_write(uint32_t blk, int band, int lane, const float* v) {
  const int odd = lane & 1;
  const int i = lane >> 1;
  const int chunk = 4 * band + (i >> 2);
  const uint32_t w = (i & 3) * 4;
#pragma unroll
  for (int jj = 0; jj < 16; ++jj) {
    const int j = (jj & 3) + 8 * (jj >> 2);
    const float send = odd ? v[j] : v[j + 4];
    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
    const __nv_bfloat162 b = __floats2bfloat162_rn(odd ? recv : v[j], odd ? v[j + 4] : recv);
    st_shared32(blk_addr(blk, j + 4 * odd, chunk) + w, *reinterpret_cast<const uint32_t*>(&b));
  }
}

// Staged block -> register block (the inverse of blk_write).
__device__ __forceinline__ void blk_read(uint32_t blk, int band, int lane, float* v) {
  const int odd = lane & 1;
  const int i = lane >> 1;
  const int chunk = 4 * band + (i >> 2);
  const uint32_t w = (i & 3) * 4;
#pragma unroll
  for (int jj = 0; jj < 16; ++jj) {
    const int j = (jj & 3) + 8 * (jj >> 2);
    const uint32_t word = ld_shared32(blk_addr(blk, j + 4 * odd, chunk) + w);
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&word));
    const float recv = __shfl_xor_sync(0xffffffffu, odd ? f.x : f.y, 1);
    v[j] = odd ? recv : f.x;
    v[j + 4] = odd ? f.y : recv;
  }
}

// One band's 32 rows x 64 bytes <-> global rows, 16 bytes a lane.  Lanes 8g .. 8g + 3 take row
// 8 it + g and lanes 8g + 4 .. 8g + 7 row 8 it + g + 4, so each group of eight lanes covers all
// 32 banks.  Rows >= rows_valid and bytes >= bytes_valid are skipped (loaded as zero).
__device__ __forceinline__ int band_row(int it, int lane) { return 8 * it + (lane >> 3) + 4 * ((lane >> 2) & 1); }

__device__ __forceinline__ void band_load(uint4 (&u)[4], int lane, const char* base, long long stride, int rows_valid,
                                          int bytes_valid) {
  const int c = lane & 3;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int r = band_row(it, lane);
    u[it] = make_uint4(0, 0, 0, 0);
    if (r < rows_valid && c * 16 < bytes_valid)
      u[it] = __ldg(reinterpret_cast<const uint4*>(base + r * stride + c * 16));
  }
}
__device__ __forceinline__ void band_put(uint32_t blk, int band, int lane, const uint4 (&u)[4]) {
  const int c = 4 * band + (lane & 3);
#pragma unroll
  for (int it = 0; it < 4; ++it) st_shared16(blk_addr(blk, band_row(it, lane), c), u[it]);
}
__device__ __forceinline__ void band_copy_out(uint32_t blk, int band, int lane, char* base, long long stride,
                                              int rows_valid, int bytes_valid) {
  const int c = lane & 3;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int r = band_row(it, lane);
    const uint4 u = ld_shared16(blk_addr(blk, r, 4 * band + c));
    if (r < rows_valid && c * 16 < bytes_valid) *reinterpret_cast<uint4*>(base + r * stride + c * 16) = u;
  }
}

// The four epilogue warps (128 threads) synchronise on named barrier 1.
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool epi_all(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred))
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void store_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Two BF16 SwiGLU products SiLU(h1) * h3 of a packed pair.
__device__ __forceinline__ uint32_t swiglu_bf16x2(uint32_t h1w, uint32_t h3w) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h1w));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h3w));
  const __nv_bfloat162 r = __floats2bfloat162_rn(a.x * sigmoid_fast(a.x) * b.x, a.y * sigmoid_fast(a.y) * b.y);
  return *reinterpret_cast<const uint32_t*>(&r);
}

// Epilogue of one pair tile for epilogue warp q (TMEM lanes 32q .. 32q + 31).
//
// Every 32-token chunk takes the same barrier steps in all four warps (the chunk count and the
// early return depend only on the tile and the CTA), so no warp is ever left at a barrier.  A
// chunk of 32 valid tokens leaves as TMA stores of whole blocks, issued by one thread
// (`issuer`); a ragged last chunk leaves with masked vector stores by each band's owner, so
// rows of the next expert segment are never touched.  `seq` counts the CTA's chunks and picks
// the chunk buffer; before each barrier after which a buffer is written again, the issuer waits
// until the stores that read that buffer have read it.
template <int EPI>
__device__ __forceinline__ void epilogue_tn(const Params& p, const TnTile& tl, uint32_t tacc, int q, int lane,
                                            uint32_t rank, uint32_t staging, int& seq, bool issuer) {
  const int nch = (tl.ntok + 31) / 32;
  const long long ldd = p.ldd;
  const int band = q & 1;
  if constexpr (EPI == EPI_SWIGLU_FWD) {
    const int fc = tl.f0 + 64 * static_cast<int>(rank);   // this CTA's 64 features
    if (fc >= p.Nout) return;
    const int fw = fc + 32 * band;
    const int bytes = max(0, min(64, (p.Nout - fw) * 2));
    const int own = q >> 1;                                 // 0: H1 band, 1: H3 band
    char* Hown = static_cast<char*>(own ? p.D1 : p.D0);
    char* A = static_cast<char*>(p.D2);
    for (int c = 0; c < nch; ++c, ++seq) {
      const int tok = tl.tok0 + 32 * c;
      const int rv = min(32, tl.ntok - 32 * c);
      const bool full = rv == 32 && p.tma_store;
      const uint32_t buf = staging + (seq & 1) * 3 * TN_BLK;
      float v[32];
      tmem_ld32(tacc + 32 * c, v);
      blk_write(buf + own * TN_BLK, band, lane, v);
      if (full) fence_async_smem();
      epi_sync();                                           // H1 and H3 blocks complete
      if (full && issuer) {
        tma_store_3d(tmd(p, 0), buf, fc, tok, 0);
        tma_store_3d(tmd(p, 1), buf + TN_BLK, fc, tok, 0);
        store_commit();
      }
      // A block, element-wise: warp q takes bytes [1024 q, 1024 q + 1024) of the three blocks.
#pragma unroll
      for (int it = 0; it < 2; ++it) {
        const uint32_t off = q * 1024 + it * 512 + lane * 16;
        const uint4 h1 = ld_shared16(buf + off);
        const uint4 h3 = ld_shared16(buf + TN_BLK + off);
        const uint4 a = make_uint4(swiglu_bf16x2(h1.x, h3.x), swiglu_bf16x2(h1.y, h3.y), swiglu_bf16x2(h1.z, h3.z),
                                   swiglu_bf16x2(h1.w, h3.w));
        st_shared16(buf + 2 * TN_BLK + off, a);
      }
      if (full) fence_async_smem();
      // Chunk buffers alternate: the next chunk's H1 / H3 go where the previous chunk's did, so
      // every store but this chunk's H1 / H3 pair must have read its block.
      if (issuer) {
        if (full) store_wait_read<1>(); else store_wait_read<0>();
      }
      epi_sync();                                           // A block complete
      if (full) {
        if (issuer) {
          tma_store_3d(tmd(p, 2), buf + 2 * TN_BLK, fc, tok, 0);
          store_commit();
        }
      } else if (bytes > 0) {
        const long long off = (static_cast<long long>(tok) * ldd + fw) * 2;
        band_copy_out(buf + own * TN_BLK, band, lane, Hown + off, ldd * 2, rv, bytes);
        if (own == 0) band_copy_out(buf + 2 * TN_BLK, band, lane, A + off, ldd * 2, rv, bytes);
      }
    }
  } else if constexpr (EPI == EPI_STORE_BF16) {
    const int fc = tl.f0 + 128 * static_cast<int>(rank);  // this CTA's 128 features: two blocks
    if (fc >= p.Nout) return;
    const int fw = fc + 32 * q;
    const int bytes = max(0, min(64, (p.Nout - fw) * 2));
    const bool second = fc + 64 < p.Nout;
    char* D = static_cast<char*>(p.D0);
    for (int c = 0; c < nch; ++c, ++seq) {
      const int tok = tl.tok0 + 32 * c;
      const int rv = min(32, tl.ntok - 32 * c);
      const bool full = rv == 32 && p.tma_store;
      const uint32_t buf = staging + (seq & 1) * 2 * TN_BLK;
      float v[32];
      tmem_ld32(tacc + 32 * c, v);
      blk_write(buf + (q >> 1) * TN_BLK, band, lane, v);
      if (full) fence_async_smem();
      if (issuer) store_wait_read<0>();                     // the previous chunk's buffer is free
      epi_sync();
      if (full) {
        if (issuer) {
          tma_store_3d(tmd(p, 0), buf, fc, tok, 0);
          if (second) tma_store_3d(tmd(p, 0), buf + TN_BLK, fc + 64, tok, 0);
          store_commit();
        }
      } else if (bytes > 0) {
        band_copy_out(buf + (q >> 1) * TN_BLK, band, lane, D + (static_cast<long long>(tok) * ldd + fw) * 2, ldd * 2,
                      rv, bytes);
      }
    }
  } else if constexpr (EPI == EPI_SWIGLU_BWD) {
    // Accumulator = dA^T.  dH1 = dA * H3 * s * (1 + H1 (1 - s)), dH3 = dA * SiLU(H1), s = sigmoid(H1).
    // Each warp brings its H1 / H3 bands in through its own bands of the dH1 / dH3 blocks (rows
    // fetched into registers one chunk ahead), then overwrites them with the results.
    const int fc = tl.f0 + 128 * static_cast<int>(rank);
    if (fc >= p.Nout) return;
    const int fw = fc + 32 * q;
    const int bytes = max(0, min(64, (p.Nout - fw) * 2));
    const bool second = fc + 64 < p.Nout;
    const int nb = p.tn_nb;
    const char* H1 = static_cast<const char*>(p.X0);
    const char* H3 = static_cast<const char*>(p.X1);
    char* dH1 = static_cast<char*>(p.D0);
    char* dH3 = static_cast<char*>(p.D1);
    uint4 r1[4], r3[4];
    {
      const long long boff = (static_cast<long long>(tl.tok0) * ldd + fw) * 2;
      band_load(r1, lane, H1 + boff, ldd * 2, min(32, tl.ntok), bytes);
      band_load(r3, lane, H3 + boff, ldd * 2, min(32, tl.ntok), bytes);
    }
    for (int c = 0; c < nch; ++c, ++seq) {
      const int tok = tl.tok0 + 32 * c;
      const int rv = min(32, tl.ntok - 32 * c);
      const bool full = rv == 32 && p.tma_store;
      const uint32_t buf = staging + (nb == 2 ? (seq & 1) : 0) * 4 * TN_BLK;
      const uint32_t b1 = buf + (q >> 1) * TN_BLK;          // dH1 half holding this warp's band
      const uint32_t b3 = b1 + 2 * TN_BLK;                  // dH3 half
      if (nb == 1) {                                        // one buffer: the last chunk's stores first
        if (issuer) store_wait_read<0>();
        epi_sync();
      }
      band_put(b1, band, lane, r1);
      band_put(b3, band, lane, r3);
      if (c + 1 < nch) {
        const long long boff = (static_cast<long long>(tok + 32) * ldd + fw) * 2;
        band_load(r1, lane, H1 + boff, ldd * 2, min(32, tl.ntok - 32 * (c + 1)), bytes);
        band_load(r3, lane, H3 + boff, ldd * 2, min(32, tl.ntok - 32 * (c + 1)), bytes);
      }
      __syncwarp();
      float da[32], h1[32], h3[32];
      blk_read(b1, band, lane, h1);
      blk_read(b3, band, lane, h3);
      __syncwarp();                                         // every lane has read the bands
      tmem_ld32(tacc + 32 * c, da);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float s = sigmoid_fast(h1[i]);
        const float d1 = da[i] * h3[i] * s * (1.0f + h1[i] * (1.0f - s));
        h1[i] = da[i] * h1[i] * s;
        da[i] = d1;
      }
      blk_write(b1, band, lane, da);
      blk_write(b3, band, lane, h1);
      if (full) fence_async_smem();
      if (issuer && nb == 2) store_wait_read<0>();
      epi_sync();
      if (full) {
        if (issuer) {
          tma_store_3d(tmd(p, 0), buf, fc, tok, 0);
          if (second) tma_store_3d(tmd(p, 0), buf + TN_BLK, fc + 64, tok, 0);
          tma_store_3d(tmd(p, 1), buf + 2 * TN_BLK, fc, tok, 0);
          if (second) tma_store_3d(tmd(p, 1), buf + 3 * TN_BLK, fc + 64, tok, 0);
          store_commit();
        }
      } else if (bytes > 0) {
        const long long off = (static_cast<long long>(tok) * ldd + fw) * 2;
        band_copy_out(b1, band, lane, dH1 + off, ldd * 2, rv, bytes);
        band_copy_out(b3, band, lane, dH3 + off, ldd * 2, rv, bytes);
      }
    }
  }
}

template <int EPI, bool GATHER = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(GATHER ? THREADS_GATHER : THREADS, 1)
    grouped_gemm_tn_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  constexpr uint32_t stage_bytes = TN_STAGE;   // 128 weight rows + 128 token rows, 128 deep in K
  uint8_t* stage_area = smem + S * stage_bytes;               // epilogue chunk buffers
  int* pair_off = reinterpret_cast<int*>(stage_area + tn_staging_bytes(EPI, p.tn_nb));
  const int poff_ints = (p.G + 1 + 63) & ~63;
  uint8_t* bar_area = reinterpret_cast<uint8_t*>(pair_off + poff_ints);
  uint64_t* full = reinterpret_cast<uint64_t*>(bar_area);
  uint64_t* empty = full + MAX_STAGES;
  uint64_t* acc_full = empty + MAX_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint64_t* landed = drain + 1;   // gathered B: stage s's copies of this CTA have landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(landed + MAX_STAGES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  constexpr uint32_t tmem_cols = 2 * TN_TOK;   // two 256-column accumulators

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // with gathered rows: the producer's expect_tx plus the relay of each CTA of the pair
      mbar_init(smem_u32(&full[s]), GATHER ? 3 : 1);
      mbar_init(smem_u32(&empty[s]), 1);
      if (GATHER) mbar_init(smem_u32(&landed[s]), 32 * GATHER_WARPS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&acc_full[b]), 1);
      mbar_init(smem_u32(&acc_empty[b]), 2 * 4 * 32);
    }
    mbar_init(smem_u32(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  // Prefix over experts of ceil(n_g / 256) token tiles (from the 128-row tile prefix).
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < p.G; base += 32) {
      const int e = base + lane;
      const int np = e < p.G ? (p.tiles[e + 1] - p.tiles[e] + 1) / 2 : 0;
      int x = np;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (e < p.G) pair_off[e] = carry + x - np;
      carry += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) pair_off[p.G] = carry;
    if (lane == 0) {
      prefetch_tmap(&p.tmA[0]);
      if (!GATHER) prefetch_tmap(&p.tmB[0]);   // gathered B has no tensor map
    }
  }
  if (warp == 1) {
    tmem_alloc2(smem_u32(tmem_slot), tmem_cols);
    tmem_relinquish2();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    // Two issuing lanes, as in the one-SM kernel: lane 0 posts the byte count (even CTA) and
    // loads A, lane 1 loads B.
    if (lane < 2) {
      uint32_t pending = 0, pend_parity = 0;
      int it = 0;
      bool ok = true;
      int wave = 0;
      TnTile tl;
      while (ok && tn_next(p, pair_off, npairs, pair, wave, tl)) {
        // This CTA's token columns [tokc, tokc + nmma / 2), loaded as one 128-row box (rows past
        // them are not read by the MMA).  Smaller boxes for ragged tiles measured slower: TMA
        // delivery per copy has a fixed cost.
        const int tokc = tl.tok0 + static_cast<int>(rank) * (tl.nmma / 2);
        const uint32_t tx = GATHER ? 2 * (2 * TN_SUB) : 2 * stage_bytes;   // gathered: A only
        for (int kb = 0; kb < tl.nk; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          if (!wait_bar2(smem_u32(&empty[s]), ph ^ 1, abort_flag, p.err)) { ok = false; break; }
          const uint32_t fb_local = smem_u32(&full[s]);
          if (leader && lane == 0) mbar_expect_tx(fb_local, tx);
          const uint32_t fb = mapa_shared(fb_local, 0);
          const uint32_t sa = smem_u32(smem + s * stage_bytes);
          const uint32_t sb = sa + 2 * TN_SUB;
          const int src = kb < p.k0_blocks ? 0 : 1;
          const int kk = (src == 0 ? kb : kb - p.k0_blocks) * TN_BK;
          pending |= 1u << s;
          pend_parity = (pend_parity & ~(1u << s)) | (ph << s);
          if (lane == 1 && GATHER) continue;   // the gather warps fill B
          if (lane == 1) {
            const CUtensorMap* tb = &p.tmB[p.nsplit ? 0 : src];
            tma_load_3d_pair(sb, tb, fb, kk, tokc, 0);
            tma_load_3d_pair(sb + TN_SUB, tb, fb, kk + BK, tokc, 0);
            continue;
          }
          if (p.a_major) {
            // MN-major weights: 64-feature blocks of 128 K rows ([block][K row][128 B])
            if (p.nsplit) {
              const int f = tl.f0 + 64 * static_cast<int>(rank);
              tma_load_3d_pair(sa, &p.tmA[0], fb, f, kk, tl.g);
              tma_load_3d_pair(sa + TN_SUB, &p.tmA[1], fb, f, kk, tl.g);
            } else {
              const int f = tl.f0 + 128 * static_cast<int>(rank);
              if (p.a_merged) {
                tma_load_4d_pair(sa, &p.tmA[src], fb, 0, kk, f / 64, tl.g);
              } else {
                tma_load_3d_pair(sa, &p.tmA[src], fb, f, kk, tl.g);
                tma_load_3d_pair(sa + TN_SUB, &p.tmA[src], fb, f + 64, kk, tl.g);
              }
            }
          } else {
            // K-major weights: two 64-deep sub-blocks of 128 feature rows ([sub-block][row][128 B])
            const int f = tl.f0 + 128 * static_cast<int>(rank);
            tma_load_3d_pair(sa, &p.tmA[src], fb, kk, f, tl.g);
            tma_load_3d_pair(sa + TN_SUB, &p.tmA[src], fb, kk + BK, f, tl.g);
          }
        }
      }
      // Drain: a stage's empty barrier completes only after the MMA consumed it, so its loads landed.
      for (int s = 0; s < S; ++s)
        if (pending & (1u << s))
          wait_bar2(smem_u32(&empty[s]), (pend_parity >> s) & 1, abort_flag, p.err, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (leader) {
      const uint32_t a_lbo = p.a_major ? TN_SUB : 16;   // MN-major: stride between 64-feature blocks
      int it = 0, tcount = 0;
      bool ok = true;
      int wave = 0;
      TnTile tl;
      for (; ok && tn_next(p, pair_off, npairs, pair, wave, tl); ++tcount) {
        const uint32_t idesc = idesc_bf16(2 * BM, tl.nmma, p.a_major, 0);
        const int buf = tcount & 1;
        const uint32_t aph = (tcount >> 1) & 1;
        ok = __all_sync(0xffffffffu, wait_bar2(smem_u32(&acc_empty[buf]), aph ^ 1, abort_flag, p.err));
        if (!ok) break;
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + buf * TN_TOK;
        for (int kb = 0; kb < tl.nk; ++kb, ++it) {
          const int s = it % S;
          const uint32_t ph = (it / S) & 1;
          ok = __all_sync(0xffffffffu, wait_bar2(smem_u32(&full[s]), ph, abort_flag, p.err));
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * stage_bytes);
          const uint32_t sb = sa + 2 * TN_SUB;
          if (lane == 0) {
#pragma unroll
            for (int kk = 0; kk < TN_BK / 16; ++kk) {
              // K-major operands: sub-block kk / 4, +32 B per K16 step inside it; MN-major: +16 rows
              const uint32_t koff = (kk >> 2) * TN_SUB + (kk & 3) * 32;
              const uint64_t ad = sdesc(sa + (p.a_major ? kk * 2048 : koff), a_lbo, 1024);
              const uint64_t bd = sdesc(sb + koff, 16, 1024);
              tc_mma2(tmem_d, ad, bd, idesc, (kb | kk) != 0);
            }
            tc_commit2_both(smem_u32(&empty[s]));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) tc_commit2_both(smem_u32(&acc_full[buf]));   // also for nk == 0 (zero tile)
        __syncwarp();
      }
      if (lane == 0) {
        tc_commit2_both(smem_u32(drain));
        wait_bar2(smem_u32(drain), 0, abort_flag, p.err, false);
      }
      __syncwarp();
    }
  } else if (GATHER && warp >= THREADS / 32 && warp < THREADS / 32 + GATHER_WARPS) {
    // ------------------------------------------------------------ token-row gather (both CTAs)
    // The dispatch gather of the X-MoE article (§2.1.2) fused into the operand ring: row r of this
    // CTA's B block is token row gather_src[gather_ids[tokc + r]], so no PFT copy of x exists.
    // Thread gt copies 16-byte chunk (gt & 7) of 64-column half ((gt >> 3) & 1) of rows
    // (gt >> 4) + 2 GATHER_WARPS i into the same 128-byte-swizzled layout a TMA box load writes (a
    // warp covers two whole rows per step: 512 contiguous bytes of x), then hands the
    // stage's completion to landed[s] (cp.async.mbarrier.arrive) and moves on: like the TMA
    // producer it runs up to a full ring ahead of the MMA.
    constexpr int RPT = 128 * 16 / (32 * GATHER_WARPS);   // rows per thread
    const int gt = threadIdx.x - THREADS;
    const int half = (gt >> 3) & 1, chunk = gt & 7, row_lo = gt >> 4;
    const __nv_bfloat16* xs = static_cast<const __nv_bfloat16*>(p.gather_src);
    int it = 0;
    bool ok = true;
    int wave = 0;
    TnTile tl;
    while (ok && tn_next(p, pair_off, npairs, pair, wave, tl)) {
      const int rows = tl.nmma / 2;                          // B rows this CTA's half of the MMA reads
      const int tokc = tl.tok0 + static_cast<int>(rank) * rows;
      const int last = p.seg[p.G] - 1;                       // rows past the segment repeat a valid row
      long long src_row[RPT];
#pragma unroll
      for (int i = 0; i < RPT; ++i) {
        const int r = max(0, min(tokc + i * (2 * GATHER_WARPS) + row_lo, last));
        src_row[i] = static_cast<long long>(p.gather_ids[r]) * p.gather_ld;
      }
      for (int kb = 0; kb < tl.nk; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1;
        ok = __all_sync(0xffffffffu, wait_bar2(smem_u32(&empty[s]), ph ^ 1, abort_flag, p.err));
        if (!ok) break;
        const uint32_t sb = smem_u32(smem + s * stage_bytes) + 2 * TN_SUB + half * TN_SUB;
        const long long col = static_cast<long long>(kb) * TN_BK + half * BK + chunk * 8;
        const bool in = col < p.gather_ld;                   // columns past d read as zeros
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
          const int row = i * (2 * GATHER_WARPS) + row_lo;
          if (row < rows) cp_async16(sb + row * 128 + ((chunk ^ (row & 7)) << 4), xs + src_row[i] + (in ? col : 0),
                                     in ? 16 : 0);
        }
        // arrives on landed[s] once every copy this thread issued so far has landed
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&landed[s])) : "memory");
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");   // no copy in flight at exit
  } else if (GATHER && warp == THREADS / 32 + GATHER_WARPS) {
    // ------------------------------------------------------------ gather relay (both CTAs)
    // Waits until a stage's gathered rows have landed, makes them visible to the tensor core's
    // (async-proxy) reads with a proxy fence, and arrives on the leader's full barrier.
    int it = 0;
    bool ok = true;
    int wave = 0;
    TnTile tl;
    while (ok && tn_next(p, pair_off, npairs, pair, wave, tl)) {
      for (int kb = 0; kb < tl.nk; ++kb, ++it) {
        const int s = it % S;
        ok = __all_sync(0xffffffffu, wait_bar2(smem_u32(&landed[s]), (it / S) & 1, abort_flag, p.err));
        if (!ok) break;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&full[s]), 0));
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const uint32_t acc_empty_leader0 = mapa_shared(smem_u32(&acc_empty[0]), 0);
    const uint32_t acc_empty_leader1 = mapa_shared(smem_u32(&acc_empty[1]), 0);
    const uint32_t staging = smem_u32(stage_area);
    const bool issuer = q == 0 && lane == 0;
    int tcount = 0, seq = 0;
    int wave = 0;
    TnTile tl;
    for (; tn_next(p, pair_off, npairs, pair, wave, tl); ++tcount) {
      const int buf = tcount & 1;
      const uint32_t aph = (tcount >> 1) & 1;
      const bool got = __all_sync(0xffffffffu, wait_bar2(smem_u32(&acc_full[buf]), aph, abort_flag, p.err));
      if (!epi_all(got)) break;   // the four warps leave together, so none waits at a barrier
      tc_fence_after();
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * TN_TOK;
      epilogue_tn<EPI>(p, tl, tacc, q, lane, rank, staging, seq, issuer);
      tc_fence_before();
      mbar_arrive_cluster(buf ? acc_empty_leader1 : acc_empty_leader0);
    }
    emit_drain(lane);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem_base, tmem_cols);
  }
}


template <int EPI, int MODE, int KBK = BK>
static int launch(Params& p, long long tile_upper_bound, const char* name, cudaStream_t stream) {
  p.mode = MODE;
  const bool staged = p.mode == KG || EPI == EPI_REDADD_BF16;
  p.stages = pick_stages(p.bn, staged, KBK);
  if (p.stages < 2) return fail(PFMOE_ERR_UNSUPPORTED, std::string(name) + ": shared-memory plan needs two stages");
  const size_t smem = smem_bytes(p.bn, p.stages, staged, KBK);
  PFMOE_TRY(smem_optin(reinterpret_cast<const void*>(&grouped_gemm_kernel<EPI, MODE, KBK>), SMEM_LIMIT, name));
  if (tile_upper_bound <= 0) return PFMOE_OK;
  long long grid = num_sms();
  if (tile_upper_bound < grid) grid = tile_upper_bound;
  PFMOE_LAUNCH(name, stream,
               (grouped_gemm_kernel<EPI, MODE, KBK><<<static_cast<int>(grid), MODE == KG ? THREADS_KG : THREADS, smem,
                                                 stream>>>(p)));
  return PFMOE_OK;
}


// Two-SM launcher for row-grouped problems: one CTA pair per two SMs of the current device.
static int max_pairs() {
  const int n = num_sms() / 2;
  return n > 0 ? n : 1;
}

// Token-as-N launcher (expert-segmented rows only).
template <int EPI, bool GATHER = false>
static int launch_tn(Params& p, long long pair_tile_upper_bound, const char* name, cudaStream_t stream) {
  p.mode = RG;
  const int stage = TN_STAGE;
  const int poff = ((p.G + 1 + 63) & ~63) * 4;
  // Two epilogue chunk buffers, unless that costs the SwiGLU backward (four blocks a chunk) its
  // third ring stage; it then runs with one buffer and a second barrier per chunk.
  p.tn_nb = 2;
  if (EPI == EPI_SWIGLU_BWD && (SMEM_LIMIT - (1024 + 512 + poff + tn_staging_bytes(EPI, 2))) / stage < 3) p.tn_nb = 1;
  const int fixed = 1024 + 512 + poff + tn_staging_bytes(EPI, p.tn_nb);
  const int st = (SMEM_LIMIT - fixed) / stage;
  if (st < 2) return fail(PFMOE_ERR_UNSUPPORTED, std::string(name) + ": too many experts for the shared-memory plan");
  p.stages = st > MAX_STAGES ? MAX_STAGES : st;
  const size_t smem = fixed + static_cast<size_t>(p.stages) * stage;
  PFMOE_TRY(smem_optin(reinterpret_cast<const void*>(&grouped_gemm_tn_kernel<EPI, GATHER>), SMEM_LIMIT, name));
  if (pair_tile_upper_bound <= 0) return PFMOE_OK;
  long long pairs = max_pairs();
  if (pair_tile_upper_bound < pairs) pairs = pair_tile_upper_bound;
  PFMOE_LAUNCH(name, stream,
               (grouped_gemm_tn_kernel<EPI, GATHER><<<static_cast<int>(2 * pairs), GATHER ? THREADS_GATHER : THREADS, smem,
                                                     stream>>>(p)));
  return PFMOE_OK;
}


// Token-tile upper bound of the token-as-N kernel: sum_e ceil(n_e / 256) <= N / 256 + E.
static long long tn_tiles_ub(int N, int E, int F, int fstep) {
  return (static_cast<long long>(N) / TN_TOK + E + 1) * ((F + fstep - 1) / fstep);
}


static Params base_params(int32_t* err) {
  Params p;
  memset(&p, 0, sizeof(p));
  p.err = err;
  p.ksplit = 1;
  return p;
}

// Split-K for the dense gate GEMMs, which have too few output tiles to fill the GPU: the part
// count (at most 8, at least 4 K blocks per part, every part non-empty) with the fewest waves of
// work on a 148-SM B200.  Depends only on the shape, so workspace sizes are host-computable.
static int choose_ksplit(long long tiles, int nk) {
  // The part count that minimises waves x K blocks per part (ties: fewer parts, less to reduce).
  const long long cap = nk / 4 > 1 ? (nk / 4 < 8 ? nk / 4 : 8) : 1;
  long long best = 1, best_cost = -1;
  for (long long ks = 1; ks <= cap; ++ks) {
    const long long kbs = (nk + ks - 1) / ks;
    const long long cost = ((tiles * ks + 147) / 148) * kbs;
    if (best_cost < 0 || cost < best_cost) { best = ks; best_cost = cost; }
  }
  const long long kbs = (nk + best - 1) / best;
  return static_cast<int>((nk + kbs - 1) / kbs);
}

__global__ void split_reduce_kernel(const float* __restrict__ parts, int nparts, long long n,
                                    const float* __restrict__ bias, int ncols, float* __restrict__ out) {
  // out = parts[0] + parts[1] + ... (fixed order) + bias[column]; n and ncols are multiples of 4.
  const long long n4 = n / 4;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float4 acc = reinterpret_cast<const float4*>(parts)[i];
    for (int s = 1; s < nparts; ++s) {
      const float4 v = reinterpret_cast<const float4*>(parts + s * n)[i];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    if (bias) {
      const int c = static_cast<int>((i * 4) % ncols);
      acc.x += bias[c]; acc.y += bias[c + 1]; acc.z += bias[c + 2]; acc.w += bias[c + 3];
    }
    reinterpret_cast<float4*>(out)[i] = acc;
  }
}

static int launch_split_reduce(const float* parts, int nparts, long long n, const float* bias, int ncols, float* out,
                               cudaStream_t s) {
  long long blocks = (n / 4 + 255) / 256;
  const long long cap = static_cast<long long>(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  PFMOE_LAUNCH("gate_split_reduce", s,
               split_reduce_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(parts, nparts, n, bias, ncols, out));
  return PFMOE_OK;
}

// Self-test of the bounded wait: one warp waits on an mbarrier nothing ever arrives at.  The wait
// must give up after limit_ns, OR PFMOE_DEV_TIMEOUT into *err and let the kernel return, leaving
// the context usable.
__global__ void wait_selftest_kernel(int32_t* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  wait_bar(smem_u32(&bar), 0, &abort_flag, err, true, limit_ns);
}

}  // namespace tc

using namespace tc;

int tc_wait_selftest(int32_t* err, unsigned long long limit_ns, cudaStream_t s) {
  PFMOE_LAUNCH("wait_selftest", s, (wait_selftest_kernel<<<1, 32, 0, s>>>(err, limit_ns)));
  return PFMOE_OK;
}

// Expert GEMMs over the PFT rows (token-as-N kernel).  seg = expert_offsets, tiles = the
// 128-row tile prefix from pft_build (the kernel derives its 256-token tile counts from it).

// H1 = X_pft W1_e, H3 = X_pft W3_e, A = SiLU(H1) * H3 (X-MoE article §2.1.2, SwiGLU expert).
int tc_ffn_gemm1(const void* x_pft, const int* seg, const int* tiles, int N, int E, int d, int h,
                 const void* w1, const void* w3, void* h1, void* h3, void* a, int32_t* err, cudaStream_t s) {
  Params p = base_params(err);
  p.nsplit = 1;
  p.Nout = h;
  p.k0_blocks = (d + TN_BK - 1) / TN_BK;
  p.seg = seg; p.tiles = tiles; p.G = E;
  p.D0 = h1; p.D1 = h3; p.D2 = a; p.ldd = h;
  p.a_major = 1;            // W1_e, W3_e [d, h]: K rows, features contiguous
  p.fstep = 128;            // 64 features of W1 and the same 64 of W3 per CTA
  PFMOE_TRY(make_tmap(&p.tmA[0], w1, h, d, E, 64, TN_BK, "w1"));
  PFMOE_TRY(make_tmap(&p.tmA[1], w3, h, d, E, 64, TN_BK, "w3"));
  PFMOE_TRY(make_tmap(&p.tmB[0], x_pft, d, N, 1, BK, 128, "x_pft"));
  PFMOE_TRY(make_out_map_tn(&p.tmD[0], h1, h, N, "h1 out"));
  PFMOE_TRY(make_out_map_tn(&p.tmD[1], h3, h, N, "h3 out"));
  PFMOE_TRY(make_out_map_tn(&p.tmD[2], a, h, N, "a out"));
  p.tma_store = 1;
  return launch_tn<EPI_SWIGLU_FWD>(p, tn_tiles_ub(N, E, h, p.fstep), "ffn_gemm1_swiglu", s);
}

// The same with the expert rows gathered from x by token_ids inside the GEMM (X_pft[r] =
// x[token_ids[r]], X-MoE article §2.1.2): the forward writes no PFT copy of x.
int tc_ffn_gemm1_gather(const void* x, const int* token_ids, const int* seg, const int* tiles, int N, int E, int d,
                        int h, const void* w1, const void* w3, void* h1, void* h3, void* a, int32_t* err,
                        cudaStream_t s) {
  Params p = base_params(err);
  p.nsplit = 1;
  p.Nout = h;
  p.k0_blocks = (d + TN_BK - 1) / TN_BK;
  p.seg = seg; p.tiles = tiles; p.G = E;
  p.D0 = h1; p.D1 = h3; p.D2 = a; p.ldd = h;
  p.a_major = 1;
  p.fstep = 128;
  p.gather_ids = token_ids; p.gather_src = x; p.gather_ld = d;
  PFMOE_TRY(make_tmap(&p.tmA[0], w1, h, d, E, 64, TN_BK, "w1"));
  PFMOE_TRY(make_tmap(&p.tmA[1], w3, h, d, E, 64, TN_BK, "w3"));
  PFMOE_TRY(make_out_map_tn(&p.tmD[0], h1, h, N, "h1 out"));
  PFMOE_TRY(make_out_map_tn(&p.tmD[1], h3, h, N, "h3 out"));
  PFMOE_TRY(make_out_map_tn(&p.tmD[2], a, h, N, "a out"));
  p.tma_store = 1;
  return launch_tn<EPI_SWIGLU_FWD, true>(p, tn_tiles_ub(N, E, h, p.fstep), "ffn_gemm1_swiglu", s);
}

// O = A W2_e.
int tc_ffn_gemm2(const void* a, const int* seg, const int* tiles, int N, int E, int d, int h, const void* w2,
                 void* out, int32_t* err, cudaStream_t s) {
  Params p = base_params(err);
  p.Nout = d;
  p.k0_blocks = (h + TN_BK - 1) / TN_BK;
  p.seg = seg; p.tiles = tiles; p.G = E;
  p.D0 = out; p.ldd = d;
  p.a_major = 1;            // W2_e [h, d]: K rows, features contiguous
  p.fstep = 2 * BM;
  p.a_merged = d % 64 == 0;
  if (p.a_merged) PFMOE_TRY(make_tmap_mn(&p.tmA[0], w2, d, h, E, TN_BK, 2, "w2"));
  else PFMOE_TRY(make_tmap(&p.tmA[0], w2, d, h, E, 64, TN_BK, "w2"));
  PFMOE_TRY(make_tmap(&p.tmB[0], a, h, N, 1, BK, 128, "a"));
  PFMOE_TRY(make_out_map_tn(&p.tmD[0], out, d, N, "out"));
  p.tma_store = 1;
  return launch_tn<EPI_STORE_BF16>(p, tn_tiles_ub(N, E, d, p.fstep), "ffn_gemm2", s);
}

// dA = dO W2_e^T, then dH1 = dA * H3 * s * (1 + H1 (1 - s)), dH3 = dA * SiLU(H1) in the epilogue.
int tc_ffn_dgrad_act(const void* dO, const int* seg, const int* tiles, int N, int E, int d, int h, const void* w2,
                     const void* h1, const void* h3, void* dh1, void* dh3, int32_t* err, cudaStream_t s) {
  Params p = base_params(err);
  p.Nout = h;
  p.k0_blocks = (d + TN_BK - 1) / TN_BK;
  p.seg = seg; p.tiles = tiles; p.G = E;
  p.X0 = h1; p.X1 = h3; p.D0 = dh1; p.D1 = dh3; p.ldd = h;
  p.a_major = 0;            // W2_e [h, d]: feature rows, K = d contiguous
  p.fstep = 2 * BM;
  PFMOE_TRY(make_tmap(&p.tmA[0], w2, d, h, E, BK, 128, "w2^T"));
  PFMOE_TRY(make_tmap(&p.tmB[0], dO, d, N, 1, BK, 128, "dO"));
  PFMOE_TRY(make_out_map_tn(&p.tmD[0], dh1, h, N, "dh1 out"));
  PFMOE_TRY(make_out_map_tn(&p.tmD[1], dh3, h, N, "dh3 out"));
  p.tma_store = 1;
  return launch_tn<EPI_SWIGLU_BWD>(p, tn_tiles_ub(N, E, h, p.fstep), "ffn_dgrad_act_swiglu_bwd", s);
}

// dX_pft = dH1 W1_e^T + dH3 W3_e^T (one K loop over both sources).
int tc_ffn_dgrad_x(const void* dh1, const void* dh3, const int* seg, const int* tiles, int N, int E, int d, int h,
                   const void* w1, const void* w3, void* dx_pft, int32_t* err, cudaStream_t s) {
  Params p = base_params(err);
  p.Nout = d;
  p.k0_blocks = (h + TN_BK - 1) / TN_BK;
  p.k1_blocks = (h + TN_BK - 1) / TN_BK;
  p.seg = seg; p.tiles = tiles; p.G = E;
  p.D0 = dx_pft; p.ldd = d;
  p.a_major = 0;            // W1_e, W3_e [d, h]: feature rows, K = h contiguous
  p.fstep = 2 * BM;
  PFMOE_TRY(make_tmap(&p.tmA[0], w1, h, d, E, BK, 128, "w1^T"));
  PFMOE_TRY(make_tmap(&p.tmA[1], w3, h, d, E, BK, 128, "w3^T"));
  PFMOE_TRY(make_tmap(&p.tmB[0], dh1, h, N, 1, BK, 128, "dh1"));
  PFMOE_TRY(make_tmap(&p.tmB[1], dh3, h, N, 1, BK, 128, "dh3"));
  PFMOE_TRY(make_out_map_tn(&p.tmD[0], dx_pft, d, N, "dx_pft out"));
  p.tma_store = 1;
  return launch_tn<EPI_STORE_BF16>(p, tn_tiles_ub(N, E, d, p.fstep), "ffn_dgrad_x", s);
}

// dW1_e = X_e^T dH1_e, dW3_e = X_e^T dH3_e (K-grouped over the expert's PFT rows).
int tc_ffn_wgrad13(const void* x_pft, const void* dh1, const void* dh3, const int* seg, int N, int E, int d, int h,
                   void* dw1, void* dw3, int32_t* err, cudaStream_t s) {
  Params p = base_params(err);
  p.mode = KG;
  p.b_major = 1;
  p.bn = h > 64 ? 256 : 128;
  p.nsplit = 1;
  p.M = d;
  p.Nout = h;
  p.seg = seg; p.G = E;
  p.D0 = dw1; p.D1 = dw3; p.ldd = h; p.d_gstride = static_cast<long long>(d) * h;
  p.a_merged = d % 64 == 0;
  p.b_merged = h % 64 == 0;
  const uint32_t bblk = (p.bn / 2) / 64;
  if (p.a_merged) PFMOE_TRY(make_tmap_mn(&p.tmA[0], x_pft, d, N, 1, BK, 2, "x_pft^T"));
  else PFMOE_TRY(make_tmap(&p.tmA[0], x_pft, d, N, 1, 64, BK, "x_pft^T"));
  if (p.b_merged) {
    PFMOE_TRY(make_tmap_mn(&p.tmB[0], dh1, h, N, 1, BK, bblk, "dh1"));
    PFMOE_TRY(make_tmap_mn(&p.tmB[1], dh3, h, N, 1, BK, bblk, "dh3"));
  } else {
    PFMOE_TRY(make_tmap(&p.tmB[0], dh1, h, N, 1, 64, BK, "dh1"));
    PFMOE_TRY(make_tmap(&p.tmB[1], dh3, h, N, 1, 64, BK, "dh3"));
  }
  PFMOE_TRY(make_out_map(&p.tmD[0], dw1, h, d, E, "dw1 out"));
  PFMOE_TRY(make_out_map(&p.tmD[1], dw3, h, d, E, "dw3 out"));
  p.tma_store = 1;
  const long long ub = static_cast<long long>(E) * ((d + BM - 1) / BM) * ((h + p.bn / 2 - 1) / (p.bn / 2));
  return launch<EPI_SPLIT_BF16, KG>(p, ub, "ffn_wgrad_w1w3", s);
}

// dW2_e = A_e^T dO_e.
int tc_ffn_wgrad2(const void* a, const void* dO, const int* seg, int N, int E, int d, int h, void* dw2,
                  int32_t* err, cudaStream_t s) {
  Params p = base_params(err);
  p.mode = KG;
  p.b_major = 1;
  p.bn = round_bn(d);
  p.M = h;
  p.Nout = d;
  p.seg = seg; p.G = E;
  p.D0 = dw2; p.ldd = d; p.d_gstride = static_cast<long long>(h) * d;
  p.a_merged = h % 64 == 0;
  p.b_merged = d % 64 == 0;
  if (p.a_merged) PFMOE_TRY(make_tmap_mn(&p.tmA[0], a, h, N, 1, BK, 2, "a^T"));
  else PFMOE_TRY(make_tmap(&p.tmA[0], a, h, N, 1, 64, BK, "a^T"));
  if (p.b_merged) PFMOE_TRY(make_tmap_mn(&p.tmB[0], dO, d, N, 1, BK, p.bn / 64, "dO"));
  else PFMOE_TRY(make_tmap(&p.tmB[0], dO, d, N, 1, 64, BK, "dO"));
  PFMOE_TRY(make_out_map(&p.tmD[0], dw2, d, h, E, "dw2 out"));
  p.tma_store = 1;
  const long long ub = static_cast<long long>(E) * ((h + BM - 1) / BM) * ((d + p.bn - 1) / p.bn);
  return launch<EPI_STORE_BF16, KG>(p, ub, "ffn_wgrad_w2", s);
}

static int gate_logits_split(int T, int d, int E) {
  const int bn = round_bn(E);
  return choose_ksplit(static_cast<long long>((T + BM - 1) / BM) * ((E + bn - 1) / bn), (d + BK - 1) / BK);
}

static int gate_wgrad_split(int T, int d, int E) {
  const int bn = round_bn(E);
  return choose_ksplit(static_cast<long long>((d + BM - 1) / BM) * ((E + bn - 1) / bn), (T + KG_BK - 1) / KG_BK);
}

size_t tc_gate_logits_ws(int T, int d, int E) {
  const int ks = gate_logits_split(T, d, E);
  return ks > 1 ? static_cast<size_t>(ks) * T * E * sizeof(float) : 0;
}

size_t tc_gate_wgrad_ws(int T, int d, int E) {
  const int ks = gate_wgrad_split(T, d, E);
  return ks > 1 ? static_cast<size_t>(ks) * d * E * sizeof(float) : 0;
}

int tc_gate_logits(const void* x, const void* wg, const float* bias, int T, int d, int E, float* logits, void* ws,
                   size_t ws_bytes, int* nparts, int32_t* err, cudaStream_t s) {
  Params p = base_params(err);
  p.mode = RG;
  p.b_major = 1;              // Wg [d, E]: K rows, E contiguous
  p.bn = round_bn(E);
  p.Nout = E;
  p.k0_blocks = (d + BK - 1) / BK;
  p.G = 1;
  p.dense_len = T;
  p.ldd = E;
  int ks = gate_logits_split(T, d, E);
  if (ws_bytes < tc_gate_logits_ws(T, d, E) || !ws) ks = 1;
  p.ksplit = ks;
  if (ks > 1) {
    p.D0 = ws;
    p.d_gstride = static_cast<long long>(T) * E;
  } else {
    p.D0 = logits;
    p.bias = bias;
  }
  PFMOE_TRY(make_tmap(&p.tmA[0], x, d, T, 1, BK, BM, "x"));
  PFMOE_TRY(make_tmap(&p.tmB[0], wg, E, d, 1, 64, 64, "wg"));
  const long long ub = static_cast<long long>((T + BM - 1) / BM) * ((E + p.bn - 1) / p.bn) * ks;
  PFMOE_TRY((launch<EPI_STORE_F32, RG>(p, ub, "gate_logits", s)));
  *nparts = ks;   // ks > 1: the top-k kernel sums the parts (and adds the bias)
  return PFMOE_OK;
}

// Gate term of the token gradient: dx[t] += sum_e dz[t, e] Wg[:, e] ([B] 训练流程, the gate's backward),
// as a dense tensor-core GEMM of the BF16 dz rows (A [T, E], K-major) against Wg (B [d, E]: N rows of
// K, read K-major, so no transpose).  The epilogue adds the product into the BF16 dx the
// token-gradient kernel wrote, with TMA reduce-add stores: every element is added once, in L2.
int tc_gate_dx(const void* dz_bf16, const void* wg, int T, int d, int E, void* dx, int32_t* err, cudaStream_t s) {
  Params p = base_params(err);
  p.mode = RG;
  p.b_major = 0;              // Wg [d, E]: rows of K
  p.bn = round_bn(d);
  p.Nout = d;
  p.k0_blocks = (E + BK - 1) / BK;
  p.G = 1;
  p.dense_len = T;
  p.ldd = d;
  p.ksplit = 1;
  p.D0 = dx;
  PFMOE_TRY(make_tmap(&p.tmA[0], dz_bf16, E, T, 1, BK, BM, "dz"));
  PFMOE_TRY(make_tmap(&p.tmB[0], wg, E, d, 1, BK, p.bn, "wg"));
  PFMOE_TRY(make_out_map(&p.tmD[0], dx, d, T, 1, "dx"));
  p.tma_store = 1;
  const long long ub = static_cast<long long>((T + BM - 1) / BM) * ((d + p.bn - 1) / p.bn);
  return launch<EPI_REDADD_BF16, RG>(p, ub, "gate_dx", s);
}

int tc_gate_wgrad(const void* x, const void* dz_bf16, int T, int d, int E, float* dwg, void* ws, size_t ws_bytes,
                  int32_t* err, cudaStream_t s) {
  Params p = base_params(err);
  p.mode = KG;
  p.b_major = 1;
  p.bn = round_bn(E);
  p.M = d;
  p.Nout = E;
  p.dense_len = T;
  p.ldd = E;
  int ks = gate_wgrad_split(T, d, E);
  if (ws_bytes < tc_gate_wgrad_ws(T, d, E) || !ws) ks = 1;
  const int nk = (T + KG_BK - 1) / KG_BK;
  const int kbs = (nk + ks - 1) / ks;
  p.kchunk = kbs * KG_BK;
  p.G = ks;
  if (ks > 1) {
    p.D0 = ws;
    p.d_gstride = static_cast<long long>(d) * E;
  } else {
    p.D0 = dwg;
    p.d_gstride = 0;
  }
  PFMOE_TRY(make_tmap(&p.tmA[0], x, d, T, 1, 64, KG_BK, "x^T"));
  PFMOE_TRY(make_tmap(&p.tmB[0], dz_bf16, E, T, 1, 64, KG_BK, "dz"));
  PFMOE_TRY(make_tmap_t(&p.tmD[0], p.D0, true, E, d, ks, 32, 32, "dwg out"));
  p.tma_store = 1;
  const long long ub = static_cast<long long>(ks) * ((d + BM - 1) / BM) * ((E + p.bn - 1) / p.bn);
  PFMOE_TRY((launch<EPI_STORE_F32, KG, KG_BK>(p, ub, "gate_wgrad", s)));
  if (ks > 1)
    PFMOE_TRY(launch_split_reduce(static_cast<const float*>(ws), ks, static_cast<long long>(d) * E, nullptr, E, dwg, s));
  return PFMOE_OK;
}

}  // namespace pfmoe
