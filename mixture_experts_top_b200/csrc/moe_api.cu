// moe_api.cu - the C ABI (include/moe.h): argument checks, workspace layout,
// and the launch sequence of each entry point.  No device memory is
// allocated here; every buffer belongs to the caller.
#include <cmath>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

thread_local std::string g_last_error;

int fail(int status, const std::string& msg) {
  g_last_error = msg;
  return status;
}

int cuda_fail(cudaError_t e, const char* where) {
  g_last_error = std::string(where) + ": " + cudaGetErrorString(e);
  return MOE_ERR_CUDA;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool is_mult8(int v) { return v >= 8 && (v % 8) == 0; }

// Checks the config; returns MOE_OK or an error status (message recorded).
int check_config(const moe_config_t* c) {
  if (c == nullptr) return fail(MOE_ERR_INVALID_ARG, "cfg is NULL");
  if (c->T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0");
  if (c->E < 1) return fail(MOE_ERR_INVALID_ARG, "E must be >= 1");
  if (c->top_k < 1 || c->top_k > c->E)
    return fail(MOE_ERR_INVALID_ARG, "top_k must satisfy 1 <= top_k <= E");
  if (c->E > 256) return fail(MOE_ERR_UNSUPPORTED, "E > 256 is not supported");
  if (c->top_k > 8) return fail(MOE_ERR_UNSUPPORTED, "top_k > 8 is not supported");
  if (!std::isfinite(c->capacity_factor))
    return fail(MOE_ERR_INVALID_ARG, "capacity_factor must be finite");
  const bool known_kind = c->expert_kind == MOE_EXPERT_LINEAR ||
                          c->expert_kind == MOE_EXPERT_RELU_MLP ||
                          c->expert_kind == MOE_EXPERT_SWIGLU;
  if (!known_kind) return fail(MOE_ERR_INVALID_ARG, "unknown expert_kind");
  if (c->act_dtype != MOE_F32 && c->act_dtype != MOE_BF16)
    return fail(MOE_ERR_INVALID_ARG, "unknown act_dtype");
  const bool pair_ok = (c->expert_kind == MOE_EXPERT_LINEAR && c->act_dtype == MOE_F32) ||
                       (c->expert_kind != MOE_EXPERT_LINEAR && c->act_dtype == MOE_BF16);
  if (!pair_ok)
    return fail(MOE_ERR_UNSUPPORTED,
                "supported: linear experts in fp32, ReLU-MLP and SwiGLU experts in bf16");
  if (!is_mult8(c->d)) return fail(MOE_ERR_UNSUPPORTED, "d must be a multiple of 8, >= 8");
  if (!is_mult8(c->d_out)) return fail(MOE_ERR_UNSUPPORTED, "d_out must be a multiple of 8, >= 8");
  if (c->expert_kind != MOE_EXPERT_LINEAR && !is_mult8(c->d_hidden))
    return fail(MOE_ERR_UNSUPPORTED, "d_hidden must be a multiple of 8, >= 8");
  if ((int64_t)c->T * c->top_k >= (int64_t)1 << 31)
    return fail(MOE_ERR_UNSUPPORTED, "T * top_k must be < 2^31");
  return MOE_OK;
}

int check_ws(const moe_config_t& c, void* ws, size_t ws_bytes) {
  if (ws == nullptr) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  const size_t need = workspace_layout(c).total;
  if (ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "workspace too small: need " + std::to_string(need) + " bytes");
  return MOE_OK;
}

#define MOE_REQUIRE(ptr)                                                      \
  do {                                                                        \
    if ((ptr) == nullptr) return fail(MOE_ERR_INVALID_ARG, #ptr " is NULL"); \
  } while (0)

// Row tensors and expert weights are moved with 16-byte vectors and TMA.
#define MOE_ALIGNED16(ptr)                                                     \
  do {                                                                         \
    if ((reinterpret_cast<uintptr_t>(ptr) & 15u) != 0)                         \
      return fail(MOE_ERR_INVALID_ARG, #ptr " must be 16-byte aligned");       \
  } while (0)

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

int act_bytes(const moe_config_t& c) { return c.act_dtype == MOE_BF16 ? 2 : 4; }

// Up and down projections (or the linear expert) on grouped rows.
// perm == nullptr: A is x_perm, the grouped rows.  Otherwise A is x (T, d)
// and grouped row r is x[perm[r]].
// pre (bf16 experts, or null): the experts' backward workspace's pre region,
// into which the up projection also writes the fp32 pre-activations.
cudaError_t run_experts(const moe_config_t& c, const void* A, const int32_t* perm,
                        const int32_t* offsets, const void* W_in, const void* W_up,
                        const void* W_out, void* y_perm, void* ws, cudaStream_t s,
                        float* pre = nullptr) {
  const WsLayout L = workspace_layout(c);
  int32_t* err = at<int32_t>(ws, L.ctrl);
  const int rows_max = c.T * c.top_k;
  if (c.expert_kind == MOE_EXPERT_LINEAR)
    return launch_linear_expert(c, static_cast<const float*>(A), offsets,
                                static_cast<const float*>(W_in), static_cast<float*>(y_perm), err,
                                s, perm);
  __nv_bfloat16* hidden = at<__nv_bfloat16>(ws, L.hidden);
  unsigned* sched = at<unsigned>(ws, L.ctrl + kCtrlGemmSched);
  const int epi = c.expert_kind == MOE_EXPERT_SWIGLU ? kEpiSwiglu : kEpiRelu;
  cudaError_t e = launch_grouped_gemm(
      epi, static_cast<const __nv_bfloat16*>(A), rows_max, c.d,
      static_cast<const __nv_bfloat16*>(W_in),
      epi == kEpiSwiglu ? static_cast<const __nv_bfloat16*>(W_up) : nullptr, c.d_hidden, c.E,
      offsets, hidden, err, sched, s, perm, c.T, nullptr, pre);
  if (e != cudaSuccess) return e;
  return launch_grouped_gemm(kEpiNone, hidden, rows_max, c.d_hidden,
                             static_cast<const __nv_bfloat16*>(W_out), nullptr, c.d_out, c.E,
                             offsets, y_perm, err, sched, s);
}

// Whether moe_forward runs the combine in the down projection's epilogue.
// Top-1 always (no y_perm at all).  Top-k: the epilogue's extra work per
// tile (write the row, count it, and for the tokens it completes read the
// other slots' rows back) must hide behind the tile's main loop, which is
// long only for a large hidden width and several tiles per CTA: on B200 the
// fused form took 0.994x the time of experts + combine at the Mixtral shape
// (d_hidden 14336), 1.002x at 64 tokens and 1.18x at E = 64, k = 6,
// d_hidden 1408.
bool fuse_combine(const moe_config_t& c) {
  if (c.expert_kind == MOE_EXPERT_LINEAR) return false;
  if (c.top_k == 1) return true;
  return c.d_hidden >= 4096 && (int64_t)c.T * c.top_k >= (int64_t)1024 * c.E;
}

// The experts and the combine.  fused (bf16 experts only): the combine is
// the down projection's epilogue.  top_k = 1: gate * row written straight
// into the token's output row, so no y_perm is written.  top_k > 1: each row
// also lands in y_perm, and the last of a token's kept rows to finish an
// output column block sums the token's rows (the up projection zeroes the
// arrival counters first).  Tokens with every slot dropped get a zero row.
// Otherwise: y_perm, then the combine kernel.
cudaError_t run_experts_combine(const moe_config_t& c, const void* x_perm,
                                const int32_t* offsets, const int32_t* perm_token,
                                const int32_t* dest, const float* gates, const void* W_in,
                                const void* W_up, const void* W_out, void* output, void* ws,
                                cudaStream_t s, bool fused) {
  const WsLayout L = workspace_layout(c);
  void* y_perm = at<void>(ws, L.y_perm);
  if (fused && c.expert_kind != MOE_EXPERT_LINEAR) {
    int32_t* err = at<int32_t>(ws, L.ctrl);
    const int rows_max = c.T * c.top_k;
    __nv_bfloat16* hidden = at<__nv_bfloat16>(ws, L.hidden);
    unsigned* sched = at<unsigned>(ws, L.ctrl + kCtrlGemmSched);
    const bool topk = c.top_k > 1;
    unsigned* arrive = topk ? at<unsigned>(ws, L.arrive) : nullptr;
    const size_t arrive_words = topk ? grouped_gemm_arrive_words(c.T, c.d_out) : 0;
    const int epi = c.expert_kind == MOE_EXPERT_SWIGLU ? kEpiSwiglu : kEpiRelu;
    cudaError_t e = launch_grouped_gemm(
        epi, static_cast<const __nv_bfloat16*>(x_perm), rows_max, c.d,
        static_cast<const __nv_bfloat16*>(W_in),
        epi == kEpiSwiglu ? static_cast<const __nv_bfloat16*>(W_up) : nullptr, c.d_hidden, c.E,
        offsets, hidden, err, sched, s, nullptr, 0, nullptr, nullptr, arrive, arrive_words);
    if (e != cudaSuccess) return e;
    const ScatterCombine sc{perm_token, gates, dest, c.T, c.top_k,
                            topk ? static_cast<float*>(y_perm) : nullptr, arrive};
    return launch_grouped_gemm(topk ? kEpiCombine : kEpiScatter, hidden, rows_max, c.d_hidden,
                               static_cast<const __nv_bfloat16*>(W_out), nullptr, c.d_out, c.E,
                               offsets, output, err, sched, s, nullptr, 0, &sc);
  }
  cudaError_t e = run_experts(c, x_perm, nullptr, offsets, W_in, W_up, W_out, y_perm, ws, s);
  if (e != cudaSuccess) return e;
  return launch_combine(c, static_cast<const float*>(y_perm), dest, gates, output, s);
}

}  // namespace

namespace {

// The library's bounded wait, made to run out: an mbarrier that nothing
// arrives on.  The wait gives up after limit_ns, records the self-test code
// on the error word and the kernel returns normally.
__global__ void wait_self_test_kernel(int32_t* err, uint64_t limit_ns) {
  pdl_wait_and_release();
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait(&bar, 0, limit_ns)) report_error(err, kDevTimeoutSelfTest);
  }
}

}  // namespace

cudaError_t launch_wait_self_test(int32_t* err, uint64_t limit_ns, cudaStream_t s) {
  return launch_kernel(wait_self_test_kernel, 1, 32, 0, s, 0, err, limit_ns);
}


WsLayout workspace_layout(const moe_config_t& c) {
  WsLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += round_up(bytes, 256);
    return o;
  };
  const size_t Tk = (size_t)c.T * (size_t)c.top_k;
  const size_t E = (size_t)c.E;
  const size_t s = (size_t)act_bytes(c);
  const size_t n_router = (size_t)std::max(1, ceil_div(c.T, kRouterTokens));
  const size_t n_chunks = (size_t)std::max(1, ceil_div(c.T, kChunkTokens));
  L.ctrl = take(256);
  L.router_part = take(n_router * E * 4);
  L.w_split = take((size_t)6 * (size_t)router_tc_width(c) * (size_t)c.d * 2);
  L.noise_z = take(router_tc_width(c) > 0 ? (size_t)c.T * E * 8 : 0);
  L.prob_mean = take(E * 4);
  L.chunk_counts = take(n_chunks * E * 4);
  L.chunk_base = take(n_chunks * E * 4);
  L.shard_prefix = take(E * 4);
  L.local_rank = take(Tk * 4);
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.dest = take(Tk * 4);
  L.perm_token = take(Tk * 4);
  L.drop_mask = take(Tk);
  L.f = take(E * 4);
  L.x_perm = take(Tk * (size_t)c.d * s);
  L.hidden = take(c.expert_kind == MOE_EXPERT_LINEAR ? 0 : Tk * (size_t)c.d_hidden * 2);
  L.y_perm = take(Tk * (size_t)c.d_out * 4);
  L.arrive = take(c.expert_kind != MOE_EXPERT_LINEAR && c.top_k > 1
                      ? grouped_gemm_arrive_words(c.T, c.d_out) * 4
                      : 0);
  const size_t nch = (size_t)route_backward_chunks(c.T, c.E);
  L.dlogits = take((size_t)c.T * E * 4);
  L.dw_part = take(nch * (size_t)c.d * E * 4);
  L.dbias_part = take(nch * E * 4);
  L.total = off;
  return L;
}

int64_t capacity_slots(float capacity_factor, int T, int k, int E) {
  const double cf = (double)capacity_factor;
  if (!(cf > 0.0)) return -1;
  return (int64_t)std::ceil(((cf * (double)T) * (double)k) / (double)E);
}

int device_sm_count() {
  static std::mutex mu;
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

cudaError_t ensure_smem_limit(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::vector<std::pair<int, const void*>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const auto& p : done)
    if (p.first == dev && p.second == kernel) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.emplace_back(dev, kernel);
  return e;
}

}  // namespace moe

using namespace moe;

extern "C" {

size_t moe_workspace_size(const moe_config_t* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return workspace_layout(*cfg).total;
}

int moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (ws == nullptr || ws_bytes < 256) return fail(MOE_ERR_WORKSPACE, "workspace NULL or < 256 bytes");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  const cudaError_t e = cudaMemsetAsync(ws, 0, 256, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_workspace_init");
}

int moe_device_status(void* ws, size_t ws_bytes, int32_t* code_out, moe_stream_t stream) {
  if (ws == nullptr || ws_bytes < 256) return fail(MOE_ERR_WORKSPACE, "workspace NULL or < 256 bytes");
  MOE_REQUIRE(code_out);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t code = 0;
  cudaError_t e = cudaMemcpyAsync(&code, ws, sizeof(code), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "moe_device_status");
  *code_out = code;
  if (code != 0) {
    e = cudaMemsetAsync(ws, 0, sizeof(code), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "moe_device_status");
    return fail(MOE_ERR_DEVICE_CHECK, "device error code " + std::to_string(code));
  }
  return MOE_OK;
}

int moe_route(const moe_config_t* cfg, const void* x, const float* W_router,
              const float* logit_bias, const float* noise, int32_t* expert_indices, float* gates,
              float* prob_mean, float* logits_out, void* ws, size_t ws_bytes,
              moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.T > 0) {
    MOE_REQUIRE(x);
    MOE_REQUIRE(expert_indices);
    MOE_REQUIRE(gates);
  }
  MOE_ALIGNED16(x);
  MOE_REQUIRE(W_router);
  MOE_REQUIRE(prob_mean);
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = workspace_layout(c);
  const cudaError_t e = launch_route(c, x, W_router, logit_bias, noise, expert_indices, gates,
                                     prob_mean, logits_out, at<float>(ws, L.router_part),
                                     at<__nv_bfloat16>(ws, L.w_split), at<int32_t>(ws, L.ctrl),
                                     reinterpret_cast<cudaStream_t>(stream),
                                     at<unsigned>(ws, L.ctrl + kCtrlRouterDone));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route");
}

}  // extern "C"

namespace {

int dispatch_entry(const moe_config_t* cfg, const moe_shard_t* sh, const void* x,
                   const int32_t* expert_indices, const float* prob_mean, int32_t* counts,
                   int32_t* offsets, int32_t* dest, int32_t* perm_token, uint8_t* drop_mask,
                   float* f, float* aux_loss, void* x_perm, void* ws, size_t ws_bytes,
                   moe_stream_t stream, const char* name) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.T > 0) {
    MOE_REQUIRE(x);
    MOE_REQUIRE(expert_indices);
    MOE_REQUIRE(dest);
    MOE_REQUIRE(perm_token);
    MOE_REQUIRE(drop_mask);
  }
  MOE_ALIGNED16(x);
  MOE_ALIGNED16(x_perm);
  if (sh == nullptr) MOE_REQUIRE(prob_mean);   // a sharded batch takes P from the records
  MOE_REQUIRE(counts);
  MOE_REQUIRE(offsets);
  MOE_REQUIRE(f);
  MOE_REQUIRE(aux_loss);
  ShardInfo shard{};
  if (sh != nullptr) {
    if (sh->world < 1 || sh->rank < 0 || sh->rank >= sh->world)
      return fail(MOE_ERR_INVALID_ARG, "shard: need 0 <= rank < world");
    if (sh->T_global < c.T || (int64_t)sh->T_global * c.top_k >= ((int64_t)1 << 31))
      return fail(MOE_ERR_INVALID_ARG, "shard: need T <= T_global and T_global * top_k < 2^31");
    if (sh->records == nullptr) return fail(MOE_ERR_INVALID_ARG, "shard->records is NULL");
    shard = ShardInfo{sh->rank, sh->world, sh->T_global, sh->records};
  }
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = workspace_layout(c);
  const cudaError_t e = launch_dispatch(
      c, x, expert_indices, prob_mean, counts, offsets, dest, perm_token, drop_mask, f, aux_loss,
      x_perm, at<int32_t>(ws, L.chunk_counts), at<int32_t>(ws, L.chunk_base),
      at<int32_t>(ws, L.local_rank), at<int32_t>(ws, L.ctrl),
      reinterpret_cast<cudaStream_t>(stream), sh != nullptr ? &shard : nullptr,
      at<int32_t>(ws, L.shard_prefix), at<unsigned>(ws, L.ctrl + kCtrlDispatchDone));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, name);
}

}  // namespace

extern "C" {

int moe_combine_backward(const moe_config_t* cfg, const void* dy, const void* y_perm,
                         const int32_t* dest, const float* gates, float* dy_perm, float* dgates,
                         moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.T > 0) {
    MOE_REQUIRE(dy);
    MOE_REQUIRE(y_perm);
    MOE_REQUIRE(dest);
    MOE_REQUIRE(gates);
    MOE_REQUIRE(dy_perm);
    MOE_REQUIRE(dgates);
  }
  MOE_ALIGNED16(dy);
  MOE_ALIGNED16(y_perm);
  MOE_ALIGNED16(dy_perm);
  const cudaError_t e = launch_combine_backward(c, dy, static_cast<const float*>(y_perm), dest,
                                                gates, dy_perm, dgates,
                                                reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_combine_backward");
}

int moe_route_backward(const moe_config_t* cfg, const void* x, const float* W_router,
                       const float* logits, const int32_t* expert_indices, const float* gates,
                       const float* f, const float* dgates, const float* daux, int32_t T_batch,
                       float* dx, float* dW_router, float* dbias, float* dlogits, void* ws,
                       size_t ws_bytes, moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.T > 0) {
    MOE_REQUIRE(x);
    MOE_REQUIRE(logits);
    MOE_REQUIRE(expert_indices);
    MOE_REQUIRE(gates);
    MOE_REQUIRE(dgates);
    MOE_REQUIRE(dx);
  }
  MOE_REQUIRE(W_router);
  MOE_REQUIRE(f);
  MOE_REQUIRE(daux);
  MOE_REQUIRE(dW_router);
  MOE_ALIGNED16(x);
  MOE_ALIGNED16(dx);
  const int Tb = T_batch > 0 ? T_batch : c.T;
  if (T_batch < 0 || (c.T > 0 && Tb < c.T))
    return fail(MOE_ERR_INVALID_ARG, "T_batch must be 0 (this call's T) or >= T");
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = workspace_layout(c);
  const cudaError_t e = launch_route_backward(
      c, x, W_router, logits, expert_indices, gates, f, dgates, daux, Tb, dx, dW_router, dbias,
      dlogits != nullptr ? dlogits : at<float>(ws, L.dlogits), at<float>(ws, L.dw_part),
      at<float>(ws, L.dbias_part), reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route_backward");
}

size_t moe_expert_backward_workspace_size(const moe_config_t* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return expert_backward_layout(*cfg).total;
}

namespace {

int expert_backward_entry(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                          const void* W_in, const void* W_up, const void* W_out,
                          const float* dy_perm, float* dx_perm, float* dW_in, float* dW_up,
                          float* dW_out, void* ws, size_t ws_bytes, moe_stream_t stream,
                          bool pre_saved) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (pre_saved && c.expert_kind == MOE_EXPERT_LINEAR)
    return fail(MOE_ERR_UNSUPPORTED, "linear experts keep no pre-activations");
  const bool swiglu = c.expert_kind == MOE_EXPERT_SWIGLU;
  const bool linear = c.expert_kind == MOE_EXPERT_LINEAR;
  MOE_REQUIRE(offsets);
  MOE_REQUIRE(W_in);
  MOE_REQUIRE(dW_in);
  if (swiglu) {
    MOE_REQUIRE(W_up);
    MOE_REQUIRE(dW_up);
  }
  if (!linear) {
    MOE_REQUIRE(W_out);
    MOE_REQUIRE(dW_out);
  }
  if (c.T > 0) {
    MOE_REQUIRE(x_perm);
    MOE_REQUIRE(dy_perm);
    MOE_REQUIRE(dx_perm);
  }
  MOE_ALIGNED16(x_perm);
  MOE_ALIGNED16(dy_perm);
  MOE_ALIGNED16(dx_perm);
  MOE_ALIGNED16(W_in);
  MOE_ALIGNED16(W_up);
  MOE_ALIGNED16(W_out);
  MOE_ALIGNED16(dW_in);
  MOE_ALIGNED16(dW_up);
  MOE_ALIGNED16(dW_out);
  if (ws == nullptr) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  const size_t need = expert_backward_layout(c).total;
  if (ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "workspace too small: need " + std::to_string(need) +
                                       " bytes (moe_expert_backward_workspace_size)");
  const cudaError_t e = launch_expert_backward(c, x_perm, offsets, W_in, W_up, W_out, dy_perm,
                                               dx_perm, dW_in, dW_up, dW_out, ws,
                                               reinterpret_cast<cudaStream_t>(stream), pre_saved);
  return e == cudaSuccess ? MOE_OK
                          : cuda_fail(e, pre_saved ? "moe_expert_ffn_backward_saved"
                                                   : "moe_expert_ffn_backward");
}

// The experts' backward workspace given to the training forward.
int check_bwd_ws(const moe_config_t& c, const void* ws, size_t ws_bytes) {
  if (ws == nullptr) return fail(MOE_ERR_WORKSPACE, "backward workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(MOE_ERR_WORKSPACE, "backward workspace must be 256-byte aligned");
  const size_t need = expert_backward_layout(c).total;
  if (ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE, "backward workspace too small: need " + std::to_string(need) +
                                       " bytes (moe_expert_backward_workspace_size)");
  return MOE_OK;
}

}  // namespace

int moe_expert_ffn_backward(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                            const void* W_in, const void* W_up, const void* W_out,
                            const float* dy_perm, float* dx_perm, float* dW_in, float* dW_up,
                            float* dW_out, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return expert_backward_entry(cfg, x_perm, offsets, W_in, W_up, W_out, dy_perm, dx_perm, dW_in,
                               dW_up, dW_out, ws, ws_bytes, stream, false);
}

int moe_expert_ffn_backward_saved(const moe_config_t* cfg, const void* x_perm,
                                  const int32_t* offsets, const void* W_in, const void* W_up,
                                  const void* W_out, const float* dy_perm, float* dx_perm,
                                  float* dW_in, float* dW_up, float* dW_out, void* ws,
                                  size_t ws_bytes, moe_stream_t stream) {
  return expert_backward_entry(cfg, x_perm, offsets, W_in, W_up, W_out, dy_perm, dx_perm, dW_in,
                               dW_up, dW_out, ws, ws_bytes, stream, true);
}

int moe_permute_backward(const moe_config_t* cfg, const float* dx_perm, const int32_t* dest,
                         const float* dx_add, float* dx, moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.T > 0) {
    MOE_REQUIRE(dx_perm);
    MOE_REQUIRE(dest);
    MOE_REQUIRE(dx);
  }
  MOE_ALIGNED16(dx_perm);
  MOE_ALIGNED16(dx_add);
  MOE_ALIGNED16(dx);
  const cudaError_t e = launch_permute_backward(c, dx_perm, dest, dx_add, dx,
                                                reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_permute_backward");
}

int moe_check_wait_timeout(void* ws, size_t ws_bytes, uint32_t limit_us, moe_stream_t stream) {
  if (ws == nullptr || ws_bytes < 256) return fail(MOE_ERR_WORKSPACE, "workspace missing or too small");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(MOE_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (limit_us == 0 || limit_us > 10000000u)
    return fail(MOE_ERR_INVALID_ARG, "limit_us must be in [1, 10^7]");
  const cudaError_t e = launch_wait_self_test(at<int32_t>(ws, 0), (uint64_t)limit_us * 1000ull,
                                              reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_check_wait_timeout");
}

int moe_gate_noise(const moe_config_t* cfg, const void* x, const float* W_noise, uint64_t seed,
                   uint64_t offset, int64_t token_base, float* noise_out, void* ws,
                   size_t ws_bytes, moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (router_tc_width(c) == 0)
    return fail(MOE_ERR_UNSUPPORTED, "moe_gate_noise: bf16 activations and E <= 64 only");
  if (c.T > 0) {
    MOE_REQUIRE(x);
    MOE_REQUIRE(noise_out);
  }
  MOE_REQUIRE(W_noise);
  MOE_ALIGNED16(x);
  if (token_base < 0) return fail(MOE_ERR_INVALID_ARG, "token_base must be >= 0");
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = workspace_layout(c);
  const cudaError_t e = launch_gate_noise(
      c, static_cast<const __nv_bfloat16*>(x), W_noise, seed, offset, (long long)token_base,
      noise_out, at<__nv_bfloat16>(ws, L.w_split), at<int32_t>(ws, L.ctrl),
      reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_gate_noise");
}

int moe_route_noisy(const moe_config_t* cfg, const void* x, const float* W_router,
                    const float* logit_bias, const float* W_noise, uint64_t seed, uint64_t offset,
                    int64_t token_base, int32_t* expert_indices, float* gates, float* prob_mean,
                    float* logits_out, float* noise_out, void* ws, size_t ws_bytes,
                    moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (router_tc_width(c) == 0)
    return fail(MOE_ERR_UNSUPPORTED, "moe_route_noisy: bf16 activations and E <= 64 only "
                                     "(elsewhere: moe_gate_noise's noise into moe_route)");
  if (c.T > 0) {
    MOE_REQUIRE(x);
    MOE_REQUIRE(expert_indices);
    MOE_REQUIRE(gates);
  }
  MOE_ALIGNED16(x);
  MOE_REQUIRE(W_router);
  MOE_REQUIRE(W_noise);
  MOE_REQUIRE(prob_mean);
  if (token_base < 0) return fail(MOE_ERR_INVALID_ARG, "token_base must be >= 0");
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = workspace_layout(c);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int tiles = 0;
  const cudaError_t e =
      c.T > 0 ? launch_route_tc_noisy(c, static_cast<const __nv_bfloat16*>(x), W_router,
                                      logit_bias, W_noise, seed, offset, (long long)token_base,
                                      expert_indices, gates, logits_out, noise_out,
                                      at<float>(ws, L.router_part),
                                      at<__nv_bfloat16>(ws, L.w_split), at<double>(ws, L.noise_z),
                                      at<int32_t>(ws, L.ctrl), s, &tiles, prob_mean,
                                      at<unsigned>(ws, L.ctrl + kCtrlRouterDone))
              : launch_prob_mean(at<float>(ws, L.router_part), 0, c.E, 0, prob_mean, s);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route_noisy");
}

int moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* expert_indices,
                 const float* prob_mean, int32_t* counts, int32_t* offsets, int32_t* dest,
                 int32_t* perm_token, uint8_t* drop_mask, float* f, float* aux_loss, void* x_perm,
                 void* ws, size_t ws_bytes, moe_stream_t stream) {
  return dispatch_entry(cfg, nullptr, x, expert_indices, prob_mean, counts, offsets, dest,
                        perm_token, drop_mask, f, aux_loss, x_perm, ws, ws_bytes, stream,
                        "moe_dispatch");
}

int moe_dispatch_count(const moe_config_t* cfg, const int32_t* expert_indices, int32_t* counts,
                       void* ws, size_t ws_bytes, moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.T > 0) MOE_REQUIRE(expert_indices);
  MOE_REQUIRE(counts);
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = workspace_layout(c);
  const cudaError_t e = launch_dispatch_count(c, expert_indices, counts,
                                              at<int32_t>(ws, L.chunk_counts),
                                              at<int32_t>(ws, L.local_rank),
                                              at<int32_t>(ws, L.ctrl),
                                              reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_dispatch_count");
}

int moe_shard_record(const moe_config_t* cfg, const int32_t* expert_indices,
                     const float* prob_mean, int32_t* record, void* ws, size_t ws_bytes,
                     moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.T > 0) MOE_REQUIRE(expert_indices);
  MOE_REQUIRE(prob_mean);
  MOE_REQUIRE(record);
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = workspace_layout(c);
  const cudaError_t e = launch_dispatch_count(c, expert_indices, record,
                                              at<int32_t>(ws, L.chunk_counts),
                                              at<int32_t>(ws, L.local_rank),
                                              at<int32_t>(ws, L.ctrl),
                                              reinterpret_cast<cudaStream_t>(stream), prob_mean);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_shard_record");
}

int moe_dispatch_shard(const moe_config_t* cfg, const moe_shard_t* shard, const void* x,
                       const int32_t* expert_indices, const float* prob_mean, int32_t* counts,
                       int32_t* offsets, int32_t* dest, int32_t* perm_token, uint8_t* drop_mask,
                       float* f, float* aux_loss, void* x_perm, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
  if (shard == nullptr) return fail(MOE_ERR_INVALID_ARG, "shard is NULL");
  return dispatch_entry(cfg, shard, x, expert_indices, prob_mean, counts, offsets, dest,
                        perm_token, drop_mask, f, aux_loss, x_perm, ws, ws_bytes, stream,
                        "moe_dispatch_shard");
}

int moe_expert_ffn(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                   const void* W_in, const void* W_up, const void* W_out, void* y_perm, void* ws,
                   size_t ws_bytes, moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  MOE_REQUIRE(offsets);
  MOE_REQUIRE(W_in);
  if (c.expert_kind == MOE_EXPERT_SWIGLU) MOE_REQUIRE(W_up);
  if (c.expert_kind != MOE_EXPERT_LINEAR) MOE_REQUIRE(W_out);
  if (c.T > 0) {
    MOE_REQUIRE(x_perm);
    MOE_REQUIRE(y_perm);
  }
  MOE_ALIGNED16(W_in);
  MOE_ALIGNED16(W_up);
  MOE_ALIGNED16(W_out);
  MOE_ALIGNED16(x_perm);
  MOE_ALIGNED16(y_perm);
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  const cudaError_t e = run_experts(c, x_perm, nullptr, offsets, W_in, W_up, W_out, y_perm, ws,
                                    reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_ffn");
}

int moe_expert_ffn_train(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                         const void* W_in, const void* W_up, const void* W_out, void* y_perm,
                         void* ws, size_t ws_bytes, void* bwd_ws, size_t bwd_ws_bytes,
                         moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.expert_kind == MOE_EXPERT_LINEAR)
    return fail(MOE_ERR_UNSUPPORTED, "linear experts keep no pre-activations");
  MOE_REQUIRE(offsets);
  MOE_REQUIRE(W_in);
  if (c.expert_kind == MOE_EXPERT_SWIGLU) MOE_REQUIRE(W_up);
  MOE_REQUIRE(W_out);
  if (c.T > 0) {
    MOE_REQUIRE(x_perm);
    MOE_REQUIRE(y_perm);
  }
  MOE_ALIGNED16(W_in);
  MOE_ALIGNED16(W_up);
  MOE_ALIGNED16(W_out);
  MOE_ALIGNED16(x_perm);
  MOE_ALIGNED16(y_perm);
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  if ((st = check_bwd_ws(c, bwd_ws, bwd_ws_bytes)) != MOE_OK) return st;
  float* pre = reinterpret_cast<float*>(static_cast<uint8_t*>(bwd_ws) +
                                        expert_backward_layout(c).pre);
  const cudaError_t e = run_experts(c, x_perm, nullptr, offsets, W_in, W_up, W_out, y_perm, ws,
                                    reinterpret_cast<cudaStream_t>(stream), pre);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_ffn_train");
}

int moe_expert_ffn_gather(const moe_config_t* cfg, const void* x, const int32_t* perm_token,
                          const int32_t* offsets, const void* W_in, const void* W_up,
                          const void* W_out, void* y_perm, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  MOE_REQUIRE(offsets);
  MOE_REQUIRE(W_in);
  if (c.expert_kind == MOE_EXPERT_SWIGLU) MOE_REQUIRE(W_up);
  if (c.expert_kind != MOE_EXPERT_LINEAR) MOE_REQUIRE(W_out);
  if (c.T > 0) {
    MOE_REQUIRE(x);
    MOE_REQUIRE(perm_token);
    MOE_REQUIRE(y_perm);
  }
  MOE_ALIGNED16(W_in);
  MOE_ALIGNED16(W_up);
  MOE_ALIGNED16(W_out);
  MOE_ALIGNED16(x);
  MOE_ALIGNED16(y_perm);
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  const cudaError_t e = run_experts(c, x, perm_token, offsets, W_in, W_up, W_out, y_perm, ws,
                                    reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_ffn_gather");
}

int moe_expert_ffn_combine(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                           const int32_t* perm_token, const int32_t* dest, const float* gates,
                           const void* W_in, const void* W_up, const void* W_out, void* output,
                           void* ws, size_t ws_bytes, moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  MOE_REQUIRE(offsets);
  MOE_REQUIRE(W_in);
  if (c.expert_kind == MOE_EXPERT_SWIGLU) MOE_REQUIRE(W_up);
  if (c.expert_kind != MOE_EXPERT_LINEAR) MOE_REQUIRE(W_out);
  if (c.T > 0) {
    MOE_REQUIRE(x_perm);
    MOE_REQUIRE(perm_token);
    MOE_REQUIRE(dest);
    MOE_REQUIRE(gates);
    MOE_REQUIRE(output);
  }
  MOE_ALIGNED16(W_in);
  MOE_ALIGNED16(W_up);
  MOE_ALIGNED16(W_out);
  MOE_ALIGNED16(x_perm);
  MOE_ALIGNED16(output);
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  if (c.T == 0) return MOE_OK;
  const cudaError_t e = run_experts_combine(c, x_perm, offsets, perm_token, dest, gates, W_in,
                                            W_up, W_out, output, ws,
                                            reinterpret_cast<cudaStream_t>(stream), true);
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_ffn_combine");
}

int moe_forward_combine_fused(const moe_config_t* cfg, int32_t* fused) {
  const int st = check_config(cfg);
  if (st != MOE_OK) return st;
  MOE_REQUIRE(fused);
  *fused = fuse_combine(*cfg) ? 1 : 0;
  return MOE_OK;
}

int moe_combine(const moe_config_t* cfg, const void* y_perm, const int32_t* dest,
                const float* gates, void* output, moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.T > 0) {
    MOE_REQUIRE(y_perm);
    MOE_REQUIRE(dest);
    MOE_REQUIRE(gates);
    MOE_REQUIRE(output);
  }
  MOE_ALIGNED16(y_perm);
  MOE_ALIGNED16(output);
  const cudaError_t e = launch_combine(c, static_cast<const float*>(y_perm), dest, gates, output,
                                       reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_combine");
}

int moe_forward(const moe_config_t* cfg, const void* x, const float* W_router,
                const float* logit_bias, const float* noise, const void* W_in, const void* W_up,
                const void* W_out, void* output, int32_t* expert_indices, float* gates,
                float* aux_loss, int32_t* counts, uint8_t* drop_mask, void* ws, size_t ws_bytes,
                moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.T > 0) {
    MOE_REQUIRE(x);
    MOE_REQUIRE(output);
    MOE_REQUIRE(expert_indices);
    MOE_REQUIRE(gates);
  }
  MOE_REQUIRE(W_router);
  MOE_REQUIRE(W_in);
  if (c.expert_kind == MOE_EXPERT_SWIGLU) MOE_REQUIRE(W_up);
  if (c.expert_kind != MOE_EXPERT_LINEAR) MOE_REQUIRE(W_out);
  MOE_REQUIRE(aux_loss);
  MOE_ALIGNED16(x);
  MOE_ALIGNED16(output);
  MOE_ALIGNED16(W_in);
  MOE_ALIGNED16(W_up);
  MOE_ALIGNED16(W_out);
  if ((st = check_ws(c, ws, ws_bytes)) != MOE_OK) return st;
  const WsLayout L = workspace_layout(c);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* P = at<float>(ws, L.prob_mean);
  int32_t* cnt = counts != nullptr ? counts : at<int32_t>(ws, L.counts);
  uint8_t* drop = drop_mask != nullptr ? drop_mask : at<uint8_t>(ws, L.drop_mask);
  int32_t* offs = at<int32_t>(ws, L.offsets);
  int32_t* dest = at<int32_t>(ws, L.dest);
  int32_t* perm = at<int32_t>(ws, L.perm_token);
  void* x_perm = at<void>(ws, L.x_perm);
  cudaError_t e = launch_route(c, x, W_router, logit_bias, noise, expert_indices, gates, P,
                               nullptr, at<float>(ws, L.router_part),
                               at<__nv_bfloat16>(ws, L.w_split), at<int32_t>(ws, L.ctrl), s,
                               at<unsigned>(ws, L.ctrl + kCtrlRouterDone));
  if (e != cudaSuccess) return cuda_fail(e, "moe_forward/route");
  e = launch_dispatch(c, x, expert_indices, P, cnt, offs, dest, perm, drop, at<float>(ws, L.f),
                      aux_loss, x_perm, at<int32_t>(ws, L.chunk_counts),
                      at<int32_t>(ws, L.chunk_base), at<int32_t>(ws, L.local_rank),
                      at<int32_t>(ws, L.ctrl), s, nullptr, nullptr,
                      at<unsigned>(ws, L.ctrl + kCtrlDispatchDone));
  if (e != cudaSuccess) return cuda_fail(e, "moe_forward/dispatch");
  // The materialised permute (one copy of each kept row, ~38 us at the
  // Mixtral shape) is far cheaper than gathering A rows inside the GEMM,
  // which re-fetches them for every output column block.
  e = run_experts_combine(c, x_perm, offs, perm, dest, gates, W_in, W_up, W_out, output, ws, s,
                          fuse_combine(c));
  if (e != cudaSuccess) return cuda_fail(e, "moe_forward/experts+combine");
  return MOE_OK;
}

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: configuration not supported";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: CUDA runtime or launch failure";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK: a kernel reported an error";
    default: return "unknown status";
  }
}

const char* moe_last_error_message(void) { return g_last_error.c_str(); }

}  // extern "C"

// ---------------------------------------------------------------------------
// moe_route_noalloc: the router for callers that cannot allocate device
// memory.  Its only scratch, the per-CTA column sums of the probabilities,
// lives in a fixed file-scope device array instead of a caller workspace.
// ---------------------------------------------------------------------------

namespace moe {
namespace {

// Fixed scratch of the allocation-free router: 65536 floats (256 KiB),
// reserved on every GPU that loads this library until the process exits.
constexpr size_t kNoAllocScratchFloats = 65536;
static __device__ __align__(256) float g_route_scratch[kNoAllocScratchFloats];

// The driver's cuCtxGetCurrent and cuCtxGetId, looked up once (nullptr if
// missing).  A context's id is unique for the life of the process, so it
// tells a context made by cudaDeviceReset from the one it replaced even if
// the new handle has the old one's value.
struct CtxIdFns {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};
const CtxIdFns& ctx_id_fns() {
  static const CtxIdFns fns = [] {
    CtxIdFns f;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 4000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    return f;
  }();
  return fns;
}

// Id of the current context, or 0 if it cannot be read.
unsigned long long current_ctx_id() {
  const CtxIdFns& f = ctx_id_fns();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (f.get_current == nullptr || f.get_id == nullptr) return 0;
  if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_route_scratch in the current device's context.  In
// host code the array's name is only a host-side stand-in, so the address
// is asked of the runtime (with that device current) the first time a
// context is seen and cached per device with that context's id.  A new
// context on the device (after cudaDeviceReset, which loads the module
// again, so the array may move) has a new id and is looked up afresh; where
// the id cannot be read, the address is looked up on every call.
cudaError_t route_scratch_address(float** out) {
  static std::mutex mu;
  static float* cached[64] = {};
  static unsigned long long cached_ctx[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_ctx_id();
  if (cached[dev] == nullptr || ctx == 0 || cached_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);   // makes the device's context current
    if (e != cudaSuccess) return e;
    cached[dev] = static_cast<float*>(p);
    cached_ctx[dev] = current_ctx_id();
  }
  *out = cached[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

extern "C" int moe_route_noalloc(const moe_config_t* cfg, const void* x, const float* W_router,
                                 const float* logit_bias, const float* noise,
                                 int32_t* expert_indices, float* gates, float* prob_mean,
                                 float* logits_out, moe_stream_t stream) {
  int st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config_t& c = *cfg;
  if (c.T > 0) {
    MOE_REQUIRE(x);
    MOE_REQUIRE(expert_indices);
    MOE_REQUIRE(gates);
  }
  MOE_ALIGNED16(x);
  MOE_REQUIRE(W_router);
  MOE_REQUIRE(prob_mean);
  const size_t need = (size_t)std::max(1, ceil_div(c.T, kRouterTokens)) * (size_t)c.E;
  if (need > kNoAllocScratchFloats)
    return fail(MOE_ERR_UNSUPPORTED,
                "moe_route_noalloc: ceil(T/32) * E = " + std::to_string(need) +
                    " exceeds its fixed scratch of " + std::to_string(kNoAllocScratchFloats) +
                    " floats; use moe_route with a workspace");
  float* scratch = nullptr;
  cudaError_t e = route_scratch_address(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "moe_route_noalloc: cudaGetSymbolAddress");
  e = launch_route(c, x, W_router, logit_bias, noise, expert_indices, gates, prob_mean,
                   logits_out, scratch, nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route_noalloc");
}
