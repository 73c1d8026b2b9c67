// C ABI of libpfmoe: host-side argument checking, workspace layout and the
// launch sequence of each step.  Every compute step runs in the library's own
// kernels (gemm_tc.cu, gemm_simt.cu, route.cu, sort.cu, rows.cu).
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <utility>
#include <string>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace pfmoe {

// ------------------------------------------------------------------ errors
static thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

int fail(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

int check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(PFMOE_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return PFMOE_OK;
}

int num_sms() {
  static std::atomic<int> cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (!n) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    n = n > 0 ? n : 1;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

int smem_optin(const void* kernel, int bytes, const char* name) {
  static std::mutex mu;
  static std::set<std::pair<int, const void*>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(PFMOE_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  std::lock_guard<std::mutex> lk(mu);
  if (done.count({dev, kernel})) return PFMOE_OK;
  // The opt-in limit covers dynamic shared memory only: the device's per-block maximum less the
  // kernel's static shared memory.
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess)
    return fail(PFMOE_ERR_CUDA, std::string(name) + ": cudaDeviceGetAttribute: " + cudaGetErrorString(e));
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess)
    return fail(PFMOE_ERR_CUDA, std::string(name) + ": cudaFuncGetAttributes: " + cudaGetErrorString(e));
  const int cap = optin - static_cast<int>(fa.sharedSizeBytes);
  if (bytes > cap) bytes = cap;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess)
    return fail(PFMOE_ERR_CUDA, std::string(name) + ": cudaFuncSetAttribute failed: " + cudaGetErrorString(e));
  done.insert({dev, kernel});
  return PFMOE_OK;
}

// ---------------------------------------------------------------- profiler
namespace {
struct ProfRec {
  const char* name;
  cudaEvent_t a, b;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_recs;
std::vector<cudaEvent_t> g_pool;
cudaEvent_t g_pending = nullptr;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}
}  // namespace

void prof_begin(const char* /*name*/, cudaStream_t s) {
  if (!g_prof_on) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_pending = take_event();
  cudaEventRecord(g_pending, s);
}

void prof_end(const char* name, cudaStream_t s) {
  if (!g_prof_on) return;
  std::lock_guard<std::mutex> lk(g_prof_mu);
  cudaEvent_t b = take_event();
  cudaEventRecord(b, s);
  g_recs.push_back({name, g_pending, b});
  g_pending = nullptr;
}

// ---------------------------------------------------------------- checking
namespace {

std::string S(const char* s) { return std::string(s); }

int need_ptr(const void* p, const char* name, bool may_be_null = false) {
  if (!p) return may_be_null ? PFMOE_OK : fail(PFMOE_ERR_ARG, S(name) + " is NULL");
  if (reinterpret_cast<uintptr_t>(p) & 15) return fail(PFMOE_ERR_ARG, S(name) + " is not 16-byte aligned");
  return PFMOE_OK;
}

int need_dtype(int dtype) {
  if (dtype != PFMOE_F32 && dtype != PFMOE_BF16) return fail(PFMOE_ERR_ARG, "dtype must be PFMOE_F32 or PFMOE_BF16");
  return PFMOE_OK;
}

int need_width(int v, const char* name, int dtype) {
  const int q = dtype == PFMOE_BF16 ? 8 : 4;
  if (v <= 0) return fail(PFMOE_ERR_ARG, S(name) + " must be positive");
  if (v % q) return fail(PFMOE_ERR_UNSUPPORTED, S(name) + " must be a multiple of " + std::to_string(q) +
                                                    " for this dtype (16-byte rows)");
  return PFMOE_OK;
}

int need_tk(int T, int k, int E) {
  if (T < 0) return fail(PFMOE_ERR_ARG, "T must be >= 0");
  if (E <= 0) return fail(PFMOE_ERR_ARG, "E must be positive");
  if (k < 1 || k > E) return fail(PFMOE_ERR_ARG, "need 1 <= k <= E");
  if (k > 32) return fail(PFMOE_ERR_UNSUPPORTED, "k must be <= 32");
  if (static_cast<long long>(T) * k >= (1LL << 31)) return fail(PFMOE_ERR_UNSUPPORTED, "T*k must fit in int32");
  return PFMOE_OK;
}

cudaStream_t st(void* s) { return static_cast<cudaStream_t>(s); }

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

struct Carve {
  char* p;
  size_t used = 0;
  explicit Carve(void* base) : p(static_cast<char*>(base)) {}
  void* take(size_t bytes) {
    void* r = p ? p + used : nullptr;
    used += align256(bytes);
    return r;
  }
};

// Backward workspace layout (shared by the size query and the call).
struct BwdWs {
  void* dO;
  float* g;
  void* dh1;
  void* dh3;
  void* da;   // FP32 path only
  void* dx_pft;
  void* wgT;
  void* dz_bf16;  // BF16 path only
  void* dwg_parts;  // BF16 path only: split-K partial sums of dWg
  size_t dwg_parts_bytes;
  size_t bytes;
};

BwdWs carve_bwd(void* base, int T, int d, int E, int h, int k, int dtype) {
  const size_t es = dtype == PFMOE_BF16 ? 2 : 4;
  const size_t N = static_cast<size_t>(T) * k;
  Carve c(base);
  BwdWs w;
  w.dO = c.take(N * d * es);
  w.g = static_cast<float*>(c.take(N * sizeof(float)));
  w.dh1 = c.take(N * h * es);
  w.dh3 = c.take(N * h * es);
  w.da = dtype == PFMOE_F32 ? c.take(N * h * es) : nullptr;
  w.dx_pft = c.take(N * d * es);
  w.wgT = c.take(static_cast<size_t>(E) * d * es);
  w.dz_bf16 = dtype == PFMOE_BF16 ? c.take(static_cast<size_t>(T) * E * 2) : nullptr;
  w.dwg_parts_bytes = dtype == PFMOE_BF16 && T > 0 ? tc_gate_wgrad_ws(T, d, E) : 0;
  w.dwg_parts = w.dwg_parts_bytes ? c.take(w.dwg_parts_bytes) : nullptr;
  w.bytes = c.used;
  return w;
}

int zero_async(void* p, size_t bytes, cudaStream_t s) {
  if (!p || !bytes) return PFMOE_OK;
  const cudaError_t e = cudaMemsetAsync(p, 0, bytes, s);
  if (e != cudaSuccess) return fail(PFMOE_ERR_CUDA, S("cudaMemsetAsync: ") + cudaGetErrorString(e));
  return PFMOE_OK;
}

}  // namespace
}  // namespace pfmoe

using namespace pfmoe;

extern "C" {

const char* moe_last_error(void) { return g_last_error.c_str(); }

int moe_abi_version(void) { return 2; }

size_t moe_route_workspace_size(int T, int d, int E, int k, int dtype) {
  if (T <= 0 || d <= 0 || E <= 0 || k <= 0 || dtype != PFMOE_BF16) return 0;
  return align256(tc_gate_logits_ws(T, d, E));
}

int moe_route(const void* x, const void* wg, const float* bias, int T, int d, int E, int k, int dtype, float* logits,
              int32_t* topk_ids, float* topk_w, void* ws, size_t ws_bytes, int32_t* err, void* stream) {
  set_error("");
  PFMOE_TRY(need_dtype(dtype));
  PFMOE_TRY(need_tk(T, k, E));
  PFMOE_TRY(need_width(d, "d", dtype));
  if (E > 1024) return fail(PFMOE_ERR_UNSUPPORTED, "E must be <= 1024");
  if (dtype == PFMOE_BF16 && E % 8) return fail(PFMOE_ERR_UNSUPPORTED, "E must be a multiple of 8 for BF16");
  if (T == 0) return PFMOE_OK;
  PFMOE_TRY(need_ptr(x, "x"));
  PFMOE_TRY(need_ptr(wg, "wg"));
  PFMOE_TRY(need_ptr(bias, "bias", true));
  PFMOE_TRY(need_ptr(logits, "logits"));
  PFMOE_TRY(need_ptr(topk_ids, "topk_ids"));
  PFMOE_TRY(need_ptr(topk_w, "topk_w"));
  PFMOE_TRY(need_ptr(ws, "ws", true));
  if (ws && ws_bytes < moe_route_workspace_size(T, d, E, k, dtype)) return fail(PFMOE_ERR_ARG, "workspace too small");
  cudaStream_t s = st(stream);
  int nparts = 1;
  if (dtype == PFMOE_BF16) {
    PFMOE_TRY(tc_gate_logits(x, wg, bias, T, d, E, logits, ws, ws_bytes, &nparts, err, s));
  } else {
    SimtGemm g{};
    g.A = static_cast<const float*>(x); g.sam = d; g.sak = 1;
    g.B = static_cast<const float*>(wg); g.sbn = 1; g.sbk = E;
    g.D = logits; g.sdm = E;
    g.bias = bias; g.G = 1; g.M = T; g.N = E; g.K = d; g.mode = 0;
    PFMOE_TRY(simt_gemm_f32(g, err, s, "gate_logits_f32"));
  }
  if (nparts > 1)   // split-K gate GEMM: the top-k kernel forms the logits from the K parts in ws
    return launch_topk(logits, static_cast<const float*>(ws), nparts, bias, T, E, k, topk_ids, topk_w, err, s);
  return launch_topk(logits, nullptr, 1, nullptr, T, E, k, topk_ids, topk_w, err, s);
}

size_t pft_build_workspace_size(int T, int E, int k) {
  if (T < 0 || E <= 0 || k <= 0) return 0;
  return align256(csort_ws_bytes(static_cast<long long>(T) * k, E));
}

int pft_build(const int32_t* topk_ids, const float* topk_w, int T, int E, int k, int32_t* tokens_per_expert,
              int32_t* expert_offsets, int32_t* token_ids, int32_t* expert_ids, float* combine_weights, int32_t* pos,
              int32_t* tile_offsets, void* ws, size_t ws_bytes, int32_t* err, void* stream) {
  set_error("");
  PFMOE_TRY(need_tk(T, k, E));
  if (E > 4096) return fail(PFMOE_ERR_UNSUPPORTED, "E must be <= 4096");
  const bool empty = T == 0;
  PFMOE_TRY(need_ptr(topk_ids, "topk_ids", empty));
  PFMOE_TRY(need_ptr(topk_w, "topk_w", empty));
  PFMOE_TRY(need_ptr(tokens_per_expert, "tokens_per_expert"));
  PFMOE_TRY(need_ptr(expert_offsets, "expert_offsets"));
  PFMOE_TRY(need_ptr(token_ids, "token_ids", empty));
  PFMOE_TRY(need_ptr(expert_ids, "expert_ids", empty));
  PFMOE_TRY(need_ptr(combine_weights, "combine_weights", empty));
  PFMOE_TRY(need_ptr(pos, "pos", empty));
  PFMOE_TRY(need_ptr(tile_offsets, "tile_offsets"));
  PFMOE_TRY(need_ptr(ws, "ws"));
  if (ws_bytes < pft_build_workspace_size(T, E, k)) return fail(PFMOE_ERR_ARG, "workspace too small");
  return pft_build_impl(topk_ids, topk_w, T, E, k, tokens_per_expert, expert_offsets, token_ids, expert_ids,
                        combine_weights, pos, tile_offsets, ws, err, st(stream));
}

int moe_dispatch(const void* x, const int32_t* pos, int T, int k, int d, int dtype, void* x_pft, int32_t* err,
                 void* stream) {
  set_error("");
  PFMOE_TRY(need_dtype(dtype));
  if (T < 0 || k < 1 || k > 32) return fail(PFMOE_ERR_ARG, "need T >= 0 and 1 <= k <= 32");
  PFMOE_TRY(need_width(d, "d", dtype));
  if (T == 0) return PFMOE_OK;
  PFMOE_TRY(need_ptr(x, "x"));
  PFMOE_TRY(need_ptr(pos, "pos"));
  PFMOE_TRY(need_ptr(x_pft, "x_pft"));
  return launch_dispatch(x, pos, T, k, d, dtype, x_pft, err, st(stream));
}

int moe_expert_ffn_gathered(const void* x, const int32_t* token_ids, const int32_t* expert_offsets,
                            const int32_t* tile_offsets, int N, int E, int d, int h, int dtype, const void* w1,
                            const void* w3, const void* w2, void* h1, void* h3, void* a, void* out, int32_t* err,
                            void* stream) {
  set_error("");
  PFMOE_TRY(need_dtype(dtype));
  if (dtype != PFMOE_BF16) return fail(PFMOE_ERR_UNSUPPORTED, "moe_expert_ffn_gathered: BF16 only");
  if (N < 0 || E <= 0) return fail(PFMOE_ERR_ARG, "need N >= 0 and E > 0");
  PFMOE_TRY(need_width(d, "d", dtype));
  PFMOE_TRY(need_width(h, "h", dtype));
  if (N == 0) return PFMOE_OK;
  PFMOE_TRY(need_ptr(x, "x"));
  PFMOE_TRY(need_ptr(token_ids, "token_ids"));
  PFMOE_TRY(need_ptr(expert_offsets, "expert_offsets"));
  PFMOE_TRY(need_ptr(tile_offsets, "tile_offsets"));
  PFMOE_TRY(need_ptr(w1, "w1"));
  PFMOE_TRY(need_ptr(w3, "w3"));
  PFMOE_TRY(need_ptr(w2, "w2"));
  PFMOE_TRY(need_ptr(h1, "h1"));
  PFMOE_TRY(need_ptr(h3, "h3"));
  PFMOE_TRY(need_ptr(a, "a"));
  PFMOE_TRY(need_ptr(out, "out"));
  cudaStream_t s = st(stream);
  PFMOE_TRY(tc_ffn_gemm1_gather(x, token_ids, expert_offsets, tile_offsets, N, E, d, h, w1, w3, h1, h3, a, err, s));
  return tc_ffn_gemm2(a, expert_offsets, tile_offsets, N, E, d, h, w2, out, err, s);
}

int moe_expert_ffn(const void* x_pft, const int32_t* expert_offsets, const int32_t* tile_offsets, int N, int E, int d,
                   int h, int dtype, const void* w1, const void* w3, const void* w2, void* h1, void* h3, void* a,
                   void* out, int32_t* err, void* stream) {
  set_error("");
  PFMOE_TRY(need_dtype(dtype));
  if (N < 0 || E <= 0) return fail(PFMOE_ERR_ARG, "need N >= 0 and E > 0");
  PFMOE_TRY(need_width(d, "d", dtype));
  PFMOE_TRY(need_width(h, "h", dtype));
  if (N == 0) return PFMOE_OK;
  PFMOE_TRY(need_ptr(x_pft, "x_pft"));
  PFMOE_TRY(need_ptr(expert_offsets, "expert_offsets"));
  PFMOE_TRY(need_ptr(tile_offsets, "tile_offsets"));
  PFMOE_TRY(need_ptr(w1, "w1"));
  PFMOE_TRY(need_ptr(w3, "w3"));
  PFMOE_TRY(need_ptr(w2, "w2"));
  PFMOE_TRY(need_ptr(h1, "h1"));
  PFMOE_TRY(need_ptr(h3, "h3"));
  PFMOE_TRY(need_ptr(a, "a"));
  PFMOE_TRY(need_ptr(out, "out"));
  cudaStream_t s = st(stream);
  if (dtype == PFMOE_BF16) {
    PFMOE_TRY(tc_ffn_gemm1(x_pft, expert_offsets, tile_offsets, N, E, d, h, w1, w3, h1, h3, a, err, s));
    return tc_ffn_gemm2(a, expert_offsets, tile_offsets, N, E, d, h, w2, out, err, s);
  }
  const long long dh = static_cast<long long>(d) * h;
  SimtGemm g{};
  g.A = static_cast<const float*>(x_pft); g.sam = d; g.sak = 1;
  g.B = static_cast<const float*>(w1); g.sbn = 1; g.sbk = h; g.b_gstride = dh;
  g.D = static_cast<float*>(h1); g.sdm = h;
  g.seg = expert_offsets; g.G = E; g.M = N; g.N = h; g.K = d; g.mode = 0;
  PFMOE_TRY(simt_gemm_f32(g, err, s, "ffn_gemm1_f32"));
  g.B = static_cast<const float*>(w3); g.D = static_cast<float*>(h3);
  PFMOE_TRY(simt_gemm_f32(g, err, s, "ffn_gemm1_f32"));
  PFMOE_TRY(simt_swiglu_fwd_f32(static_cast<const float*>(h1), static_cast<const float*>(h3), static_cast<float*>(a),
                                static_cast<long long>(N) * h, s));
  SimtGemm g2{};
  g2.A = static_cast<const float*>(a); g2.sam = h; g2.sak = 1;
  g2.B = static_cast<const float*>(w2); g2.sbn = 1; g2.sbk = d; g2.b_gstride = dh;
  g2.D = static_cast<float*>(out); g2.sdm = d;
  g2.seg = expert_offsets; g2.G = E; g2.M = N; g2.N = d; g2.K = h; g2.mode = 0;
  return simt_gemm_f32(g2, err, s, "ffn_gemm2_f32");
}

int moe_combine(const void* out, const int32_t* pos, const float* topk_w, int T, int k, int d, int dtype, void* y,
                int32_t* err, void* stream) {
  set_error("");
  PFMOE_TRY(need_dtype(dtype));
  if (T < 0 || k < 1 || k > 32) return fail(PFMOE_ERR_ARG, "need T >= 0 and 1 <= k <= 32");
  PFMOE_TRY(need_width(d, "d", dtype));
  if (T == 0) return PFMOE_OK;
  PFMOE_TRY(need_ptr(out, "out"));
  PFMOE_TRY(need_ptr(pos, "pos"));
  PFMOE_TRY(need_ptr(topk_w, "topk_w"));
  PFMOE_TRY(need_ptr(y, "y"));
  return launch_combine(out, pos, topk_w, T, k, d, dtype, y, err, st(stream));
}

size_t moe_backward_workspace_size(int T, int d, int E, int h, int k, int dtype) {
  if (T < 0 || d <= 0 || E <= 0 || h <= 0 || k <= 0 || (dtype != PFMOE_F32 && dtype != PFMOE_BF16)) return 0;
  return carve_bwd(nullptr, T, d, E, h, k, dtype).bytes;
}

int moe_backward(const void* dy, const void* x, const void* wg, const float* topk_w, const int32_t* topk_ids,
                 const int32_t* pos, const int32_t* expert_offsets, const int32_t* tile_offsets, const void* x_pft,
                 const void* h1, const void* h3, const void* a, const void* out, const void* w1, const void* w3,
                 const void* w2, int T, int d, int E, int h, int k, int dtype, void* dx, float* dwg, void* dw1,
                 void* dw3, void* dw2, float* dlogits, void* ws, size_t ws_bytes, int32_t* err, void* stream) {
  set_error("");
  PFMOE_TRY(need_dtype(dtype));
  PFMOE_TRY(need_tk(T, k, E));
  PFMOE_TRY(need_width(d, "d", dtype));
  PFMOE_TRY(need_width(h, "h", dtype));
  if (dtype == PFMOE_BF16 && E % 8) return fail(PFMOE_ERR_UNSUPPORTED, "E must be a multiple of 8 for BF16");
  const bool empty = T == 0;
  const void* must[] = {wg, w1, w3, w2, dwg, dw1, dw3, dw2};
  const char* must_n[] = {"wg", "w1", "w3", "w2", "dwg", "dw1", "dw3", "dw2"};
  for (int i = 0; i < 8; ++i) PFMOE_TRY(need_ptr(must[i], must_n[i]));
  const void* tok[] = {dy, x, topk_w, topk_ids, pos, expert_offsets, tile_offsets, x_pft, h1, h3, a, out, dx, dlogits, ws};
  const char* tok_n[] = {"dy", "x", "topk_w", "topk_ids", "pos", "expert_offsets", "tile_offsets", "x_pft",
                         "h1", "h3", "a", "out", "dx", "dlogits", "ws"};
  for (int i = 0; i < 15; ++i) PFMOE_TRY(need_ptr(tok[i], tok_n[i], empty));
  cudaStream_t s = st(stream);
  const size_t es = dtype == PFMOE_BF16 ? 2 : 4;
  if (empty) {
    // No tokens: every weight gradient is exactly zero.
    PFMOE_TRY(zero_async(dw1, static_cast<size_t>(E) * d * h * es, s));
    PFMOE_TRY(zero_async(dw3, static_cast<size_t>(E) * d * h * es, s));
    PFMOE_TRY(zero_async(dw2, static_cast<size_t>(E) * d * h * es, s));
    return zero_async(dwg, static_cast<size_t>(d) * E * sizeof(float), s);
  }
  if (ws_bytes < moe_backward_workspace_size(T, d, E, h, k, dtype)) return fail(PFMOE_ERR_ARG, "workspace too small");
  const BwdWs w = carve_bwd(ws, T, d, E, h, k, dtype);
  const int N = T * k;

  PFMOE_TRY(launch_combine_bwd(dy, out, pos, topk_w, T, k, d, dtype, w.dO, w.g, err, s));
  if (dtype == PFMOE_BF16) {
    PFMOE_TRY(tc_ffn_dgrad_act(w.dO, expert_offsets, tile_offsets, N, E, d, h, w2, h1, h3, w.dh1, w.dh3, err, s));
    PFMOE_TRY(tc_ffn_dgrad_x(w.dh1, w.dh3, expert_offsets, tile_offsets, N, E, d, h, w1, w3, w.dx_pft, err, s));
    PFMOE_TRY(tc_ffn_wgrad13(x_pft, w.dh1, w.dh3, expert_offsets, N, E, d, h, dw1, dw3, err, s));
    PFMOE_TRY(tc_ffn_wgrad2(a, w.dO, expert_offsets, N, E, d, h, dw2, err, s));
    // dx = sum of the token's dX_pft rows (and dz, dlogits); then the gate term on the tensor cores
    PFMOE_TRY(launch_token_grad(w.dx_pft, pos, w.g, topk_w, topk_ids, nullptr, T, k, d, E, dtype, dx, dlogits,
                                w.dz_bf16, err, s));
    PFMOE_TRY(tc_gate_dx(w.dz_bf16, wg, T, d, E, dx, err, s));
    return tc_gate_wgrad(x, w.dz_bf16, T, d, E, dwg, w.dwg_parts, w.dwg_parts_bytes, err, s);
  }
  // FP32 path on the CUDA cores.
  const long long dh = static_cast<long long>(d) * h;
  float* dO = static_cast<float*>(w.dO);
  float* da = static_cast<float*>(w.da);
  float* dh1 = static_cast<float*>(w.dh1);
  float* dh3 = static_cast<float*>(w.dh3);
  float* dxp = static_cast<float*>(w.dx_pft);
  SimtGemm g{};
  // dA = dO W2_e^T : B(n = h, k = d) = W2[e][n][k]
  g.A = dO; g.sam = d; g.sak = 1;
  g.B = static_cast<const float*>(w2); g.sbn = d; g.sbk = 1; g.b_gstride = dh;
  g.D = da; g.sdm = h; g.seg = expert_offsets; g.G = E; g.M = N; g.N = h; g.K = d; g.mode = 0;
  PFMOE_TRY(simt_gemm_f32(g, err, s, "ffn_dgrad_act_f32"));
  PFMOE_TRY(simt_swiglu_bwd_f32(da, static_cast<const float*>(h1), static_cast<const float*>(h3), dh1, dh3,
                                static_cast<long long>(N) * h, s));
  // dX = dH1 W1_e^T + dH3 W3_e^T : B(n = d, k = h) = W1[e][n][k]
  g = SimtGemm{};
  g.A = dh1; g.sam = h; g.sak = 1;
  g.B = static_cast<const float*>(w1); g.sbn = h; g.sbk = 1; g.b_gstride = dh;
  g.D = dxp; g.sdm = d; g.seg = expert_offsets; g.G = E; g.M = N; g.N = d; g.K = h; g.mode = 0;
  PFMOE_TRY(simt_gemm_f32(g, err, s, "ffn_dgrad_x_f32"));
  g.A = dh3; g.B = static_cast<const float*>(w3); g.beta = 1.f;
  PFMOE_TRY(simt_gemm_f32(g, err, s, "ffn_dgrad_x_f32"));
  // dW1 = X_e^T dH1, dW3 = X_e^T dH3 : K grouped over the expert's rows
  g = SimtGemm{};
  g.A = static_cast<const float*>(x_pft); g.sam = 1; g.sak = d;
  g.B = dh1; g.sbn = 1; g.sbk = h;
  g.D = static_cast<float*>(dw1); g.sdm = h; g.d_gstride = dh;
  g.seg = expert_offsets; g.G = E; g.M = d; g.N = h; g.K = N; g.mode = 1;
  PFMOE_TRY(simt_gemm_f32(g, err, s, "ffn_wgrad_w1w3_f32"));
  g.B = dh3; g.D = static_cast<float*>(dw3);
  PFMOE_TRY(simt_gemm_f32(g, err, s, "ffn_wgrad_w1w3_f32"));
  // dW2 = A_e^T dO
  g = SimtGemm{};
  g.A = static_cast<const float*>(a); g.sam = 1; g.sak = h;
  g.B = dO; g.sbn = 1; g.sbk = d;
  g.D = static_cast<float*>(dw2); g.sdm = d; g.d_gstride = dh;
  g.seg = expert_offsets; g.G = E; g.M = h; g.N = d; g.K = N; g.mode = 1;
  PFMOE_TRY(simt_gemm_f32(g, err, s, "ffn_wgrad_w2_f32"));
  PFMOE_TRY(launch_transpose(wg, d, E, dtype, w.wgT, s));
  PFMOE_TRY(launch_token_grad(w.dx_pft, pos, w.g, topk_w, topk_ids, w.wgT, T, k, d, E, dtype, dx, dlogits, nullptr,
                              err, s));
  // dWg = x^T dz (dense, K = T)
  g = SimtGemm{};
  g.A = static_cast<const float*>(x); g.sam = 1; g.sak = d;
  g.B = dlogits; g.sbn = 1; g.sbk = E;
  g.D = dwg; g.sdm = E; g.G = 1; g.M = d; g.N = E; g.K = T; g.mode = 1;
  return simt_gemm_f32(g, err, s, "gate_wgrad_f32");
}

size_t rbd_plan_workspace_size(int T, int k, int E, int experts_per_device, int devices_per_node) {
  if (T < 0 || k <= 0 || E <= 0 || experts_per_device <= 0 || devices_per_node <= 0) return 0;
  const long long epn = static_cast<long long>(experts_per_device) * devices_per_node;
  if (epn > E || E % epn) return 0;
  return align256(rbd_ws_bytes(T, k, E, static_cast<int>(E / epn)));
}

int rbd_plan(const int32_t* topk_ids, int T, int k, int E, int experts_per_device, int devices_per_node,
             int32_t* pilots_per_node, int32_t* node_offsets, int32_t* pilot_token, int32_t* pilot_node,
             int32_t* pilot_device, int32_t* replica_offsets, int32_t* replica_expert, int32_t* assign_pilot,
             int32_t* counts, void* ws, size_t ws_bytes, int32_t* err, void* stream) {
  set_error("");
  PFMOE_TRY(need_tk(T, k, E));
  if (experts_per_device <= 0 || devices_per_node <= 0)
    return fail(PFMOE_ERR_ARG, "experts_per_device and devices_per_node must be positive");
  const long long epn = static_cast<long long>(experts_per_device) * devices_per_node;
  if (epn > E || E % epn) return fail(PFMOE_ERR_ARG, "E must be a multiple of experts_per_device*devices_per_node");
  const int n_nodes = static_cast<int>(E / epn);
  if (n_nodes > 4096) return fail(PFMOE_ERR_UNSUPPORTED, "at most 4096 nodes");
  const bool empty = T == 0;
  PFMOE_TRY(need_ptr(topk_ids, "topk_ids", empty));
  PFMOE_TRY(need_ptr(pilots_per_node, "pilots_per_node"));
  PFMOE_TRY(need_ptr(node_offsets, "node_offsets"));
  PFMOE_TRY(need_ptr(pilot_token, "pilot_token", empty));
  PFMOE_TRY(need_ptr(pilot_node, "pilot_node", empty));
  PFMOE_TRY(need_ptr(pilot_device, "pilot_device", empty));
  PFMOE_TRY(need_ptr(replica_offsets, "replica_offsets"));
  PFMOE_TRY(need_ptr(replica_expert, "replica_expert", empty));
  PFMOE_TRY(need_ptr(assign_pilot, "assign_pilot", empty));
  PFMOE_TRY(need_ptr(counts, "counts"));
  PFMOE_TRY(need_ptr(ws, "ws"));
  if (ws_bytes < rbd_plan_workspace_size(T, k, E, experts_per_device, devices_per_node))
    return fail(PFMOE_ERR_ARG, "workspace too small");
  return rbd_plan_impl(topk_ids, T, k, E, experts_per_device, devices_per_node, pilots_per_node, node_offsets,
                       pilot_token, pilot_node, pilot_device, replica_offsets, replica_expert, assign_pilot, counts,
                       ws, err, st(stream));
}

int moe_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = on != 0;
  return PFMOE_OK;
}

void moe_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_recs) {
    cudaEventSynchronize(r.b);
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
}

int moe_profile_read(char* names, int name_stride, int max_entries, double* total_ms, int* launches) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  std::vector<std::string> order;
  std::map<std::string, std::pair<double, int>> agg;
  for (auto& r : g_recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return -1;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return -1;
    auto it = agg.find(r.name);
    if (it == agg.end()) {
      order.push_back(r.name);
      agg[r.name] = {ms, 1};
    } else {
      it->second.first += ms;
      it->second.second += 1;
    }
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  int n = 0;
  for (const auto& nm : order) {
    if (n >= max_entries) break;
    if (names && name_stride > 0) {
      std::strncpy(names + static_cast<size_t>(n) * name_stride, nm.c_str(), name_stride - 1);
      names[static_cast<size_t>(n) * name_stride + name_stride - 1] = '\0';
    }
    if (total_ms) total_ms[n] = agg[nm].first;
    if (launches) launches[n] = agg[nm].second;
    ++n;
  }
  return n;
}

int moe_selftest_wait_timeout(int32_t* err, unsigned long long limit_ns, void* stream) {
  set_error("");
  PFMOE_TRY(need_ptr(err, "err"));
  if (limit_ns < 1000000ull || limit_ns > 5000000000ull) return fail(PFMOE_ERR_ARG, "limit_ns must be in [1e6, 5e9]");
  return tc_wait_selftest(err, limit_ns, st(stream));
}

}  // extern "C"
