// moe_internal.h - host-side declarations shared by the library's .cu files.
#pragma once

#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include <algorithm>
#include <utility>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Smallest number of tokens a router CTA owns (every router configuration
// uses a whole multiple of it, so ceil(T / kRouterTokens) bounds the number
// of router CTAs and sizes the per-CTA partial sums), and the tokens of one
// dispatch chunk.
constexpr int kRouterTokens = 32;
constexpr int kChunkTokens = 256;

// Workspace regions, byte offsets from the workspace base (each 256-aligned).
struct WsLayout {
  size_t ctrl;           // int32 error word (+ padding)
  size_t router_part;    // (router CTAs, E) fp32 per-CTA column sums of probs
  size_t w_split;        // (6, EP, d) bf16: W_router (and W_noise) split for the tensor-core router
  size_t noise_z;        // (T, E) fp64: the noisy gate's draws (moe_route_noisy)
  size_t prob_mean;      // (E) fp32, moe_forward only
  size_t chunk_counts;   // (chunks, E) int32
  size_t chunk_base;     // (chunks, E) int32
  size_t shard_prefix;   // (E) int32: earlier ranks' slots per expert (sharded batch)
  size_t local_rank;     // (T*k) int32 position of a slot inside its chunk
  size_t counts;         // (E) int32           -- moe_forward intermediates
  size_t offsets;        // (E+1) int32
  size_t dest;           // (T*k) int32
  size_t perm_token;     // (T*k) int32
  size_t drop_mask;      // (T*k) uint8
  size_t f;              // (E) fp32
  size_t x_perm;         // (T*k, d) act
  size_t hidden;         // (T*k, d_hidden) bf16
  size_t y_perm;         // (T*k, d_out) fp32
  size_t arrive;         // (T, d_out / 256) uint32: the top-k combine's arrival counters
  size_t dlogits;        // (T, E) fp32: moe_route_backward's logit gradient
  size_t dw_part;        // (chunks, d, E) fp32: per-chunk partial dW_router
  size_t dbias_part;     // (chunks, E) fp32
  size_t total;
};

WsLayout workspace_layout(const moe_config_t& c);

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Per-device properties cached on first use.
int device_sm_count();

// The driver's cuTensorMapEncodeTiled, looked up once (nullptr if missing).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Expert columns of the tensor-core router for this configuration (E padded
// to 16, 32 or 64), or 0 where the fp32 SIMT router runs instead (fp32
// activations, or E > 64).
inline int router_tc_width(const moe_config_t& c) {
  if (c.act_dtype != MOE_BF16 || c.E > 64) return 0;
  return c.E <= 16 ? 16 : (c.E <= 32 ? 32 : 64);
}

// Sets a kernel's dynamic shared-memory limit once per (device, kernel).
cudaError_t ensure_smem_limit(const void* kernel, int bytes);

// Launches `kern` with programmatic stream serialization (the kernel may be
// scheduled while its predecessor drains; it waits for it in-kernel) and, if
// cluster > 0, an explicit 1-D cluster of that many CTAs (0: no cluster
// attribute).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster > 0) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Launchers; each returns cudaSuccess or the launch error.
// w_split (6 * router_tc_width(c) * d bf16) selects the tensor-core router
// where router_tc_width(c) > 0; nullptr always runs the SIMT router.  err is
// the workspace error word and done its tile counter (both may be nullptr
// with w_split == nullptr).
cudaError_t launch_route(const moe_config_t& c, const void* x, const float* W_router,
                         const float* bias, const float* noise, int32_t* idx, float* gates,
                         float* prob_mean, float* logits_out, float* router_part,
                         __nv_bfloat16* w_split, int32_t* err, cudaStream_t s,
                         unsigned* done = nullptr);
// The workspace's control block (first 256 bytes, cleared by
// moe_workspace_init): the error word at byte 0, the router's tile counter
// at byte kCtrlRouterDone, the pair GEMM's tile counter (two unsigned) at
// byte kCtrlGemmSched and the dispatch count's chunk counter at byte
// kCtrlDispatchDone, each on its own 64-byte line.  The kernels leave every
// counter at 0.
constexpr size_t kCtrlRouterDone = 64;
constexpr size_t kCtrlGemmSched = 128;
constexpr size_t kCtrlDispatchDone = 192;
// The noisy gate's noise (router_tc.cu): noise_out (T, E) fp32 =
// z(token_base + t, e) * softplus(x @ W_noise); bf16 x and E <= 64 only.
cudaError_t launch_gate_noise(const moe_config_t& c, const __nv_bfloat16* x, const float* W_noise,
                              uint64_t seed, uint64_t offset, long long token_base,
                              float* noise_out, __nv_bfloat16* w_split, int32_t* err,
                              cudaStream_t s);
// Tensor-core router (router_tc.cu): logits, softmax, top-k, gates, one row
// of probability column sums per 128-token tile (*tiles_out = rows) and,
// from the last tile to finish, P_e into prob_mean; `done` is a counter that
// must be 0 before the launch and is 0 again after it.
cudaError_t launch_route_tc(const moe_config_t& c, const __nv_bfloat16* x, const float* W_router,
                            const float* bias, const float* noise, int32_t* idx, float* gates,
                            float* logits_out, float* router_part, __nv_bfloat16* w_split,
                            int32_t* err, cudaStream_t s, int* tiles_out, float* prob_mean,
                            unsigned* done);

// The tensor-core router with the noisy gate's noise made in the kernel:
// noise = z(token_base + t, e) * softplus(x @ W_noise) added after the bias;
// noise_out (T, E) fp32 or nullptr receives the noise drawn.  w_split holds
// 6 * router_tc_width(c) * d bf16, noise_z (T, E) fp64 the draws z.
cudaError_t launch_route_tc_noisy(const moe_config_t& c, const __nv_bfloat16* x,
                                  const float* W_router, const float* bias, const float* W_noise,
                                  uint64_t seed, uint64_t offset, long long token_base,
                                  int32_t* idx, float* gates, float* logits_out, float* noise_out,
                                  float* router_part, __nv_bfloat16* w_split, double* noise_z,
                                  int32_t* err, cudaStream_t s, int* tiles_out, float* prob_mean,
                                  unsigned* done);
// P_e = (the column-sum rows of router_part added in fp64) / T (router.cu).
cudaError_t launch_prob_mean(const float* router_part, int rows, int E, int T, float* prob_mean,
                             cudaStream_t s);

// A batch split over `world` ranks in contiguous token blocks, rank order:
// every rank's exchange record (world, 2E+1) int32 on the device (E slot
// counts, E probability means as fp32 bits, the token count), and the whole
// batch's token count.
struct ShardInfo {
  int rank, world, T_global;
  const int32_t* records;
};
cudaError_t launch_dispatch(const moe_config_t& c, const void* x, const int32_t* idx,
                            const float* prob_mean, int32_t* counts, int32_t* offsets,
                            int32_t* dest, int32_t* perm_token, uint8_t* drop_mask, float* f,
                            float* aux, void* x_perm, int32_t* chunk_counts, int32_t* chunk_base,
                            int32_t* local_rank, int32_t* err, cudaStream_t s,
                            const ShardInfo* shard = nullptr, int32_t* shard_prefix = nullptr,
                            unsigned* done = nullptr);
// The per-expert slot counts of `idx` (T, top_k) into counts (E); with
// prob_mean != nullptr, counts is a (2E+1) exchange record: the counts,
// the fp32 bits of prob_mean and T.
cudaError_t launch_dispatch_count(const moe_config_t& c, const int32_t* idx, int32_t* counts,
                                  int32_t* chunk_counts, int32_t* local_rank, int32_t* err,
                                  cudaStream_t s, const float* prob_mean = nullptr);

cudaError_t launch_combine(const moe_config_t& c, const float* y_perm, const int32_t* dest,
                           const float* gates, void* out, cudaStream_t s);

// perm != nullptr: grouped row r is row perm[r] of x_perm, a (T, d) tensor.
cudaError_t launch_linear_expert(const moe_config_t& c, const float* x_perm,
                                 const int32_t* offsets, const float* W, float* y_perm,
                                 int32_t* err, cudaStream_t s, const int32_t* perm = nullptr);

// Grouped bf16 GEMM on tcgen05: for every expert e, rows [offsets[e],
// offsets[e+1]) of A (rows_max, K) times B_e (K, N) -> out rows, with a fused
// epilogue.  epi: 0 = none (fp32 output), 1 = ReLU (bf16 output), 2 = SwiGLU
// (bf16 output; B0 = gate, B1 = up; each output column pairs one gate and
// one up column), 3 = the top-1 combine (bf16 output rows of tokens: grouped
// row r writes gates[t] * acc into row t = rows[r]; tokens with dest[t] < 0
// get a zero row), 4 = the top-k combine (fp32 rows into y, as epi 0; the
// last of a token's kept rows to finish a column block sums the token's rows
// in slot order into its bf16 output row; tokens with every slot dropped get
// a zero row).
enum GemmEpilogue { kEpiNone = 0, kEpiRelu = 1, kEpiSwiglu = 2, kEpiScatter = 3, kEpiCombine = 4 };
struct ScatterCombine {
  const int32_t* rows;   // (rows) token of each grouped row (perm_token)
  const float* gates;    // (T, top_k) the slots' gates
  const int32_t* dest;   // (T, top_k) the slots' grouped rows, -1 if dropped
  int T;
  int top_k;             // 1 for kEpiScatter
  float* y;              // kEpiCombine: (rows, N) fp32 expert rows (y_perm)
  // kEpiCombine: grouped_gemm_arrive_words(T, N) arrival counters, 0 at
  // launch (the up projection's `clear` zeroes them).
  unsigned* arrive;
};
// Arrival counters kEpiCombine needs for T tokens and N output columns.
size_t grouped_gemm_arrive_words(int T, int N);

// perm != nullptr (ReLU / SwiGLU only): grouped row r of A is row perm[r] of
// A, an (a_rows, K) tensor, fetched by TMA row gathers (the permute fused into
// the up projection's operand load).
// sched: the workspace's tile counter (two unsigned, 0 before the launch and
// left at 0), used where the CTA-pair kernel runs.
// pre (kEpiSwiglu / kEpiRelu only, or null): also write every kept row's fp32
// pre-activations into the experts' backward layout (the `pre` region of its
// workspace, expert_backward_layout), for moe_expert_ffn_backward_saved.
// clear (or null): clear_words words the epilogue warps set to 0 before
// their first tile (the next launch's kEpiCombine arrival counters).
cudaError_t launch_grouped_gemm(int epi, const __nv_bfloat16* A, int rows_max, int K,
                                const __nv_bfloat16* B0, const __nv_bfloat16* B1, int N, int E,
                                const int32_t* offsets, void* out, int32_t* err, unsigned* sched,
                                cudaStream_t s, const int32_t* perm = nullptr, int a_rows = 0,
                                const ScatterCombine* sc = nullptr, float* pre = nullptr,
                                unsigned* clear = nullptr, size_t clear_words = 0);

// Experts' backward (expert_backward.cu, grouped_gemm_bwd.cu).  The bf16
// GEMMs work on a padded grouped layout: each expert's rows rounded up to a
// multiple of kBwdPadRows, zero rows after its own.
constexpr int kBwdPadRows = 64;
// Hidden units per block of the backward's stored pre-activations (the M of a pair tile).
constexpr int kBwdPreBlock = 256;
// Rows of the padded layout for at most rows_max grouped rows.
int expert_backward_pad_rows(int rows_max, int E);
// Workspace of moe_expert_ffn_backward: error word; padded rows Xp (bf16),
// dYp (bf16); pre-activations [A | B] (fp32), their gradients [dA | dB] and
// H (bf16).
struct ExpertBwdLayout {
  size_t ctrl, xp, dyp, pre, dab, hid, total;
};
ExpertBwdLayout expert_backward_layout(const moe_config_t& c);
// pre_saved: the workspace's pre region already holds the pre-activations
// (written by the training forward); they are not recomputed, and the pack
// launch zeroes their padding rows.
cudaError_t launch_expert_backward(const moe_config_t& c, const void* x_perm,
                                   const int32_t* offsets, const void* W_in, const void* W_up,
                                   const void* W_out, const float* dy_perm, float* dx_perm,
                                   float* dW_in, float* dW_up, float* dW_out, void* ws,
                                   cudaStream_t s, bool pre_saved = false);
cudaError_t launch_expert_backward_gemms(const moe_config_t& c, const int32_t* offsets,
                                         const __nv_bfloat16* xp, const __nv_bfloat16* dyp,
                                         const __nv_bfloat16* W_in, const __nv_bfloat16* W_up,
                                         const __nv_bfloat16* W_out, float* pre,
                                         __nv_bfloat16* dab, __nv_bfloat16* hid, float* dx_perm,
                                         float* dW_in, float* dW_up, float* dW_out, int32_t* err,
                                         cudaStream_t s, bool pre_saved = false);
// dx (T, d) = dx_add (or 0) + sum over kept slots j of dx_perm[dest[t, j]].
cudaError_t launch_permute_backward(const moe_config_t& c, const float* dx_perm,
                                    const int32_t* dest, const float* dx_add, float* dx,
                                    cudaStream_t s);

// Routing backward (backward.cu).
int route_backward_chunks(int T, int E);
cudaError_t launch_combine_backward(const moe_config_t& c, const void* dy, const float* y_perm,
                                    const int32_t* dest, const float* gates, float* dy_perm,
                                    float* dgates, cudaStream_t s);
cudaError_t launch_route_backward(const moe_config_t& c, const void* x, const float* W,
                                  const float* logits, const int32_t* idx, const float* gates,
                                  const float* f, const float* dgates, const float* daux,
                                  int T_batch, float* dx, float* dW, float* dbias,
                                  float* dlogits, float* dw_part, float* dbias_part,
                                  cudaStream_t s);
// One bounded mbarrier wait that nothing completes; after limit_ns the kernel
// writes the self-test code to err and returns (moe_api.cu).
cudaError_t launch_wait_self_test(int32_t* err, uint64_t limit_ns, cudaStream_t s);
// Host-side capacity: ceil(((cf * T) * k) / E) in fp64, or -1 for no limit.
int64_t capacity_slots(float capacity_factor, int T, int k, int E);

}  // namespace moe
