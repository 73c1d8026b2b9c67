// Internal launchers of libpfmoe (not part of the C ABI).  Each returns a
// PFMOE_* status and launches on `s` without synchronising.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pfmoe {

// ---- tensor-core grouped GEMMs (BF16 operands, FP32 accumulation), gemm_tc.cu
int tc_ffn_gemm1(const void* x_pft, const int* seg, const int* tiles, int N, int E, int d, int h,
                 const void* w1, const void* w3, void* h1, void* h3, void* a, int32_t* err, cudaStream_t s);
int tc_ffn_gemm1_gather(const void* x, const int* token_ids, const int* seg, const int* tiles, int N, int E, int d,
                        int h, const void* w1, const void* w3, void* h1, void* h3, void* a, int32_t* err,
                        cudaStream_t s);
int tc_gate_dx(const void* dz_bf16, const void* wg, int T, int d, int E, void* dx, int32_t* err, cudaStream_t s);
int tc_ffn_gemm2(const void* a, const int* seg, const int* tiles, int N, int E, int d, int h, const void* w2,
                 void* out, int32_t* err, cudaStream_t s);
int tc_ffn_dgrad_act(const void* dO, const int* seg, const int* tiles, int N, int E, int d, int h, const void* w2,
                     const void* h1, const void* h3, void* dh1, void* dh3, int32_t* err, cudaStream_t s);
int tc_ffn_dgrad_x(const void* dh1, const void* dh3, const int* seg, const int* tiles, int N, int E, int d, int h,
                   const void* w1, const void* w3, void* dx_pft, int32_t* err, cudaStream_t s);
int tc_ffn_wgrad13(const void* x_pft, const void* dh1, const void* dh3, const int* seg, int N, int E, int d, int h,
                   void* dw1, void* dw3, int32_t* err, cudaStream_t s);
int tc_ffn_wgrad2(const void* a, const void* dO, const int* seg, int N, int E, int d, int h, void* dw2,
                  int32_t* err, cudaStream_t s);
// Dense gate GEMMs split K over a workspace (sizes below; 0 = no split) and reduce deterministically.
size_t tc_gate_logits_ws(int T, int d, int E);
size_t tc_gate_wgrad_ws(int T, int d, int E);
// Gate logits X Wg (+ bias).  When the GEMM is split along K (ws large enough), the K parts are
// left in ws ([*nparts][T][E] FP32) for launch_topk to sum; otherwise *nparts = 1 and logits holds
// the result.
int tc_gate_logits(const void* x, const void* wg, const float* bias, int T, int d, int E, float* logits, void* ws,
                   size_t ws_bytes, int* nparts, int32_t* err, cudaStream_t s);
int tc_gate_wgrad(const void* x, const void* dz_bf16, int T, int d, int E, float* dwg, void* ws, size_t ws_bytes,
                  int32_t* err, cudaStream_t s);

// ---- FP32 SIMT grouped GEMM, gemm_simt.cu
// D(m, n) = beta * D(m, n) + sum_k A(m, k) B(n, k) (+ bias[n]).
// A(m, k) = A[m * sam + k * sak], B(n, k) = B[n * sbn + k * sbk], D(m, n) = D[m * sdm + n].
// mode 0 (rows grouped): group g covers A/D rows [seg[g], seg[g+1]); B advances by b_gstride per group.
// mode 1 (K grouped): group g reduces over k in [seg[g], seg[g+1]) (A, B row offsets) and D advances by d_gstride.
// seg == null: one group, rows [0, M) (mode 0) or k in [0, K) (mode 1).
struct SimtGemm {
  const float* A; long long sam, sak;
  const float* B; long long sbn, sbk, b_gstride;
  float* D; long long sdm, d_gstride;
  const float* bias;
  const int* seg;
  int G, M, N, K, mode;
  float beta;
};
int simt_gemm_f32(const SimtGemm& g, int32_t* err, cudaStream_t s, const char* name);
int simt_swiglu_fwd_f32(const float* h1, const float* h3, float* a, long long n, cudaStream_t s);
int simt_swiglu_bwd_f32(const float* da, const float* h1, const float* h3, float* dh1, float* dh3, long long n,
                        cudaStream_t s);

// ---- routing, route.cu
// Top-k softmax over logits [T][E].  With parts != null the logits are first formed as
// parts[0] + ... + parts[nparts-1] (+ bias), in that order, and written to logits.
int tc_wait_selftest(int32_t* err, unsigned long long limit_ns, cudaStream_t s);
int launch_topk(float* logits, const float* parts, int nparts, const float* bias, int T, int E, int k, int32_t* ids,
                float* w, int32_t* err, cudaStream_t s);

// ---- stable counting sort, PFT, RBD: sort.cu
// Stable counting sort of n keys in [0, K): chunk histograms + scan.  n may be read
// from the device (n_dev != null) with n_max bounding it.
size_t csort_ws_bytes(long long n_max, int K);
int pft_build_impl(const int32_t* ids, const float* w, int T, int E, int k, int32_t* tpe, int32_t* offsets,
                   int32_t* token_ids, int32_t* expert_ids, float* cw, int32_t* pos, int32_t* tile_offsets,
                   void* ws, int32_t* err, cudaStream_t s);
size_t rbd_ws_bytes(int T, int k, int E, int n_nodes);
int rbd_plan_impl(const int32_t* ids, int T, int k, int E, int epd, int dpn, int32_t* pilots_per_node,
                  int32_t* node_offsets, int32_t* pilot_token, int32_t* pilot_node, int32_t* pilot_device,
                  int32_t* replica_offsets, int32_t* replica_expert, int32_t* assign_pilot, int32_t* counts,
                  void* ws, int32_t* err, cudaStream_t s);

// ---- row kernels, rows.cu (dtype 0 = float, 1 = bf16)
int launch_dispatch(const void* x, const int32_t* pos, int T, int k, int d, int dtype, void* x_pft, int32_t* err,
                    cudaStream_t s);
int launch_combine(const void* out, const int32_t* pos, const float* w, int T, int k, int d, int dtype, void* y,
                   int32_t* err, cudaStream_t s);
int launch_combine_bwd(const void* dy, const void* out, const int32_t* pos, const float* w, int T, int k, int d,
                       int dtype, void* dO, float* g, int32_t* err, cudaStream_t s);
int launch_transpose(const void* in, int rows, int cols, int dtype, void* out, cudaStream_t s);
int launch_token_grad(const void* dx_pft, const int32_t* pos, const float* g, const float* w, const int32_t* ids,
                      const void* wgT, int T, int k, int d, int E, int dtype, void* dx, float* dlogits,
                      void* dz_bf16, int32_t* err, cudaStream_t s);

}  // namespace pfmoe
