/*
 * pfmoe.h -- C ABI of the padding-free MoE layer library (libpfmoe.so), sm_100a.
 *
 * The library computes one MoE layer with padding-free token buffers (PFT) on
 * one GPU: top-k softmax gate, PFT build, dispatch, SwiGLU expert FFN as a
 * grouped GEMM over variable-length expert segments, weighted combine, the
 * full backward, and the redundancy-bypassing-dispatch (RBD) pilot plan.
 *
 * Sources (page title + section):
 *   [A] X-MoE article (adg.csdn.net), §2.1.1 "PFT数据结构创新", §2.1.2 "跨平台核函数优化",
 *       §2.2.1 "分层冗余消除算法".
 *   [B] "5.4 MoE模型在分布式训练中的应用" (aiknowledge.cn), section 训练流程.
 *   [C] Reading notes "【论文】略读笔记90-前沿-可扩展 MoE 训练", sections 需求 / 创新.
 *
 * Conventions shared by every entry point
 *   - Every data pointer is a DEVICE pointer owned by the caller.  The library
 *     never allocates device memory and keeps no state between calls (except the
 *     optional profiler below).  Scratch memory is passed in as (ws, ws_bytes);
 *     query its size with the matching *_workspace_size function.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronises with the host.  Data-dependent
 *     counts (tokens per expert, GEMM tiles, pilots) stay on the device.
 *   - Tensors are dense row-major.  `dtype` selects the storage type of the
 *     activations and weights: PFMOE_BF16 (bfloat16, FP32 accumulate) or
 *     PFMOE_F32.  Logits, routing weights, dlogits and dWg are always float32;
 *     indices are int32.
 *   - Device pointers must be 16-byte aligned.  For PFMOE_BF16, d, h and E must
 *     be multiples of 8 (16-byte rows); for PFMOE_F32, multiples of 4.
 *   - Return value: PFMOE_OK, or an error code with a message available from
 *     moe_last_error() (thread-local).  Argument errors are detected on the host
 *     before anything is launched.
 *   - `err` (nullable) is a device int32 the kernels OR error bits into
 *     (PFMOE_DEV_*).  The caller zeroes it; nothing traps.  After a device error
 *     bit is set the outputs of that call are unspecified.
 */
#ifndef PFMOE_H
#define PFMOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PFMOE_API __attribute__((visibility("default")))
#else
#define PFMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum { PFMOE_OK = 0, PFMOE_ERR_ARG = 1, PFMOE_ERR_UNSUPPORTED = 2, PFMOE_ERR_CUDA = 3 };
enum { PFMOE_F32 = 0, PFMOE_BF16 = 1 };

/* Device error bits written into *err. */
enum {
  PFMOE_DEV_BAD_EXPERT_ID = 1, /* a routed expert id outside [0, E) */
  PFMOE_DEV_BAD_POS = 2,       /* a PFT row index outside [0, T*k) */
  PFMOE_DEV_TIMEOUT = 4,       /* a bounded on-chip wait gave up (the kernel returned early) */
  PFMOE_DEV_NONFINITE = 8      /* a NaN gate logit was seen (it ranks below every number), or a
                                  token's largest logit is +inf or -inf (its weights are undefined) */
};

/* Rows per grouped-GEMM M tile.  Expert e owns ceil(n_e / PFMOE_TILE_ROWS) tiles. */
#define PFMOE_TILE_ROWS 128

/* Last error message of the calling thread ("" if none). */
PFMOE_API const char* moe_last_error(void);
/* Library ABI version (increments on incompatible changes). */
PFMOE_API int moe_abi_version(void);

/*
 * moe_route -- gate logits and top-k selection ([B] 训练流程 step a; [C] 需求: large top-k).
 *   x [T,d] (dtype), wg [d,E] (dtype), bias [E] float32 or NULL (added to the logits).
 *   logits [T,E] float32 out: z = x wg + bias, FP32 accumulation.
 *   topk_ids [T,k] int32 out: per token the k largest logits, descending; equal
 *     logits are ordered by the lower expert index.  Selection is decided on the
 *     float32 logits written to `logits`.
 *   topk_w [T,k] float32 out: softmax over the k selected logits (sums to 1).
 *   ws (nullable): moe_route_workspace_size(...) bytes.  With it, the BF16 gate GEMM
 *   splits its K dimension over more SMs and sums the parts in a fixed order (the
 *   result does not depend on the split); without it the GEMM runs unsplit.
 *   Requires 1 <= k <= E, k <= 32, E <= 1024.
 */
PFMOE_API size_t moe_route_workspace_size(int T, int d, int E, int k, int dtype);
PFMOE_API int moe_route(const void* x, const void* wg, const float* bias, int T, int d, int E, int k, int dtype,
                        float* logits, int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes, int32_t* err,
                        void* stream);

/*
 * pft_build -- the padding-free token buffer's index fields ([A] §2.1.1).
 *   The N = T*k assignments a = t*k + j are sorted stably by expert id: rows of
 *   expert e are [expert_offsets[e], expert_offsets[e+1]) with tokens ascending.
 *   No capacity, no padding, no dropping (every assignment gets one row).
 *   topk_ids [T,k] int32, topk_w [T,k] float32 in.
 *   tokens_per_expert [E], expert_offsets [E+1], token_ids [N], expert_ids [N]
 *   (int32), combine_weights [N] float32, pos [T,k] int32 (row of assignment
 *   (t,j)), tile_offsets [E+1] int32 (prefix over experts of
 *   ceil(n_e / PFMOE_TILE_ROWS): the grouped-GEMM tile list) out.
 *   ws: pft_build_workspace_size(T, E, k) bytes.  Out-of-range ids set
 *   PFMOE_DEV_BAD_EXPERT_ID and are left out.  Requires E <= 4096.
 */
PFMOE_API size_t pft_build_workspace_size(int T, int E, int k);
PFMOE_API int pft_build(const int32_t* topk_ids, const float* topk_w, int T, int E, int k,
              int32_t* tokens_per_expert, int32_t* expert_offsets, int32_t* token_ids,
              int32_t* expert_ids, float* combine_weights, int32_t* pos, int32_t* tile_offsets,
              void* ws, size_t ws_bytes, int32_t* err, void* stream);

/*
 * pft_build_no_ws -- pft_build for callers that cannot allocate device memory.
 *   No counterpart in the X-MoE pages: this is a service of this library.
 *   Some callers cannot hand pft_build a workspace -- for example a process whose
 *   device memory is all carved out by another pool at start-up, or a fixed C
 *   interface that passes only input and output pointers.  This entry point takes
 *   the same inputs and outputs as pft_build and gives the same results, but
 *   uses a scratch array built into the library (PFMOE_PFT_NO_WS_SCRATCH_BYTES
 *   bytes of device memory that every GPU loading the library holds until the
 *   process exits).  It allocates nothing.
 *   Limit: pft_build_workspace_size(T, E, k) must not exceed
 *   PFMOE_PFT_NO_WS_SCRATCH_BYTES (for example T*k up to 260096 with E = 1024, 1046528 with E = 256);
 *   larger shapes return PFMOE_ERR_UNSUPPORTED with a message naming both sizes.
 *   The first call on a device looks up the array's device address (once, with
 *   that device current); make that first call before any stream capture (a
 *   first call on a capturing stream returns PFMOE_ERR_UNSUPPORTED).  The address
 *   is cached for the life of the process: do not call this entry point on a
 *   device after cudaDeviceReset of that device.
 *   All calls on a device share the array and it keeps the last call's contents
 *   (nothing has to start at zero); calls that overlap on the GPU race on it.
 */
#define PFMOE_PFT_NO_WS_SCRATCH_BYTES (1u << 20)
PFMOE_API int pft_build_no_ws(const int32_t* topk_ids, const float* topk_w, int T, int E, int k,
                              int32_t* tokens_per_expert, int32_t* expert_offsets, int32_t* token_ids,
                              int32_t* expert_ids, float* combine_weights, int32_t* pos, int32_t* tile_offsets,
                              int32_t* err, void* stream);

/*
 * moe_dispatch -- PFT.x ([A] §2.1.2 gather): row pos[t,j] of x_pft [T*k, d]
 *   receives token row x[t].  Equivalent to x_pft[r] = x[token_ids[r]]; it is
 *   computed token-major so that every x row is read once.
 */
PFMOE_API int moe_dispatch(const void* x, const int32_t* pos, int T, int k, int d, int dtype, void* x_pft,
                 int32_t* err, void* stream);

/*
 * moe_expert_ffn -- SwiGLU expert FFN over the expert-sorted buffer ([A] §2.1.2
 *   per-expert GEMM without padding; expert form: [B] 参数分布的不均匀性).
 *   For expert e and its rows R_e = [expert_offsets[e], expert_offsets[e+1]):
 *     H1 = X W1_e, H3 = X W3_e, A = SiLU(H1) * H3, O = A W2_e,   SiLU(u) = u sigmoid(u).
 *   x_pft [N,d]; w1, w3 [E,d,h]; w2 [E,h,d]; h1, h3, a [N,h] out (saved for the
 *   backward); out [N,d] out.  tile_offsets from pft_build.  N = T*k.
 */
PFMOE_API int moe_expert_ffn(const void* x_pft, const int32_t* expert_offsets, const int32_t* tile_offsets,
                   int N, int E, int d, int h, int dtype, const void* w1, const void* w3, const void* w2,
                   void* h1, void* h3, void* a, void* out, int32_t* err, void* stream);

/*
 * moe_expert_ffn_gathered -- moe_expert_ffn with the dispatch gather fused into the
 *   first expert GEMM ([A] §2.1.2: the expert reads its rows by token id; [A] §1 and
 *   §2.1.1: dispatch buffers dominate activation memory).  Row r of the expert input
 *   is x[token_ids[r]] (x [T,d]; token_ids [N] from pft_build), read straight into the
 *   GEMM's operand ring: no [N,d] copy of x is written.  Same outputs, layout and
 *   tolerance as moe_expert_ffn.  BF16 only (PFMOE_ERR_UNSUPPORTED otherwise); d and
 *   h multiples of 8.  token_ids must hold valid token indices (< T) for all N rows:
 *   the kernel does not check them.
 */
PFMOE_API int moe_expert_ffn_gathered(const void* x, const int32_t* token_ids, const int32_t* expert_offsets,
                            const int32_t* tile_offsets, int N, int E, int d, int h, int dtype, const void* w1,
                            const void* w3, const void* w2, void* h1, void* h3, void* a, void* out, int32_t* err,
                            void* stream);

/*
 * moe_combine -- y[t] = sum_{j<k} topk_w[t,j] * out[pos[t,j]] ([A] §2.1.1
 *   combine_weights; [B] 训练流程 step d), summed in slot order in float32 and
 *   rounded once.  Deterministic (no atomics).  y [T,d] out.
 */
PFMOE_API int moe_combine(const void* out, const int32_t* pos, const float* topk_w, int T, int k, int d, int dtype,
                void* y, int32_t* err, void* stream);

/*
 * moe_backward -- gradients of the whole layer ([B] 训练流程: backward along the
 *   reverse path), given dy [T,d] = dL/dy and the forward's saved tensors.
 *   Outputs: dx [T,d] (dtype), dwg [d,E] float32, dw1, dw3 [E,d,h] and dw2
 *   [E,h,d] (dtype; experts with no rows get exact zeros), dlogits [T,E]
 *   float32 (non-zero only at the selected experts:
 *   dz_{t,ids[t,j]} = w_j (g_j - sum_l w_l g_l), g_j = <dy_t, out[pos[t,j]]>).
 *   ws: moe_backward_workspace_size(T, d, E, h, k, dtype) bytes.
 */
PFMOE_API size_t moe_backward_workspace_size(int T, int d, int E, int h, int k, int dtype);
PFMOE_API int moe_backward(const void* dy, const void* x, const void* wg, const float* topk_w, const int32_t* topk_ids,
                 const int32_t* pos, const int32_t* expert_offsets, const int32_t* tile_offsets,
                 const void* x_pft, const void* h1, const void* h3, const void* a, const void* out,
                 const void* w1, const void* w3, const void* w2, int T, int d, int E, int h, int k, int dtype,
                 void* dx, float* dwg, void* dw1, void* dw3, void* dw2, float* dlogits,
                 void* ws, size_t ws_bytes, int32_t* err, void* stream);

/*
 * rbd_plan -- redundancy-bypassing dispatch plan ([A] §2.2.1), indexing only.
 *   Virtual map: device(e) = e / experts_per_device, node(e) = e / (experts_per_device *
 *   devices_per_node); n_nodes = E / (experts_per_device * devices_per_node) (E must be a
 *   multiple).  One pilot per (token, distinct node among its k experts), ordered
 *   by node then token.  Pmax = T * min(k, n_nodes).
 *   pilots_per_node [n_nodes], node_offsets [n_nodes+1], pilot_token [Pmax],
 *   pilot_node [Pmax], pilot_device [Pmax] (device of the pilot's lowest-id
 *   replica), replica_offsets [Pmax+1] (CSR over pilots), replica_expert [T*k]
 *   (each pilot's experts ascending), assign_pilot [T,k] (pilot carrying (t,j)),
 *   counts [2] = {num_pilots P, number of distinct (token, device) pairs}.
 *   Entries past P are left untouched.  ws: rbd_plan_workspace_size bytes.
 */
PFMOE_API size_t rbd_plan_workspace_size(int T, int k, int E, int experts_per_device, int devices_per_node);
PFMOE_API int rbd_plan(const int32_t* topk_ids, int T, int k, int E, int experts_per_device, int devices_per_node,
             int32_t* pilots_per_node, int32_t* node_offsets, int32_t* pilot_token, int32_t* pilot_node,
             int32_t* pilot_device, int32_t* replica_offsets, int32_t* replica_expert, int32_t* assign_pilot,
             int32_t* counts, void* ws, size_t ws_bytes, int32_t* err, void* stream);

/*
 * Kernel profiler.  While enabled, every kernel the library launches is
 * bracketed by two CUDA events recorded on its launch stream.  moe_profile_read
 * synchronises on those events and returns, per kernel name, the number of
 * launches and their summed device time in milliseconds.  Not thread-safe
 * against concurrent launches from several host threads.
 *   moe_profile_read: names receives up to max_entries NUL-terminated names,
 *   name_stride bytes apart; returns the number of entries (or -1 on error).
 */
PFMOE_API int moe_profile_enable(int on);
PFMOE_API void moe_profile_reset(void);
PFMOE_API int moe_profile_read(char* names, int name_stride, int max_entries, double* total_ms, int* launches);

/*
 * Test support, not part of the layer (the X-MoE pages have no counterpart).
 * moe_selftest_wait_timeout launches one warp that waits, with the bounded mbarrier wait
 * every GEMM of this library uses, on a barrier nothing ever arrives at.  After limit_ns
 * nanoseconds (1 ms .. 5 s) the wait gives up, ORs PFMOE_DEV_TIMEOUT into *err (device
 * memory) and the kernel returns; the CUDA context stays usable.  This lets a test drive
 * the timeout path without faulting or hanging the GPU.  Asynchronous on `stream`.
 * Errors: PFMOE_ERR_ARG for a null err or a limit outside the range.
 */
PFMOE_API int moe_selftest_wait_timeout(int32_t* err, unsigned long long limit_ns, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* PFMOE_H */
