/*
 * moe.h - C ABI of the B200 (sm_100a) forward pass of a sparsely-gated
 * Mixture-of-Experts layer.
 *
 * What the layer computes (pages cited by title and section):
 *   [MLG] "Mixture-of-Experts Routing - LLM Internals" (mlgrind.dev),
 *         sections "Algorithm", "Inputs", "Expected Return Format",
 *         "Edge cases and conventions", "Follow-up".
 *   [PFD] "Mixture of Experts: the Sparsely-Gated Layer" (paperfordummies.in),
 *         sections "The one formula", "The code",
 *         "Switch: top-1, one loss, and a rate limit".
 *   [EB]  "Sparsely-gated Mixture of Experts (MoE)" (Eli Bendersky's website),
 *         section "A Minimal Numpy Implementation".
 *
 *   logits  = x @ W_router (+ logit_bias) (+ noise)            fp32   [MLG Algorithm 1; PFD The code]
 *   probs   = softmax(logits) over the E experts                fp32   [MLG Algorithm 1]
 *   indices = the top_k experts by descending logit, ties to the lower index
 *                                                                       [MLG Algorithm 2, Edge cases]
 *   gates   = softmax of the chosen top_k logits (rows sum to 1)      [MLG Algorithm 2]
 *   dispatch: slots (t, j) in token order; slot position p = earlier slots
 *             on the same expert; kept iff p < cap,
 *             cap = ceil(((capacity_factor * T) * top_k) / E) in fp64
 *                                                  [MLG Follow-up; PFD Switch, The code]
 *   y_t     = sum over kept slots j of gates[t,j] * expert_{indices[t,j]}(x_t)
 *             (a dropped slot adds 0; gates are not renormalised)   [MLG Algorithm 3; PFD Switch]
 *   aux     = E * sum_e f_e * P_e, f_e = slots routed to e / (T*top_k)
 *             (before capacity), P_e = mean_t probs[t,e]             [MLG Algorithm 4]
 *
 * Experts (weights in the pages' x @ W orientation, row-major (E, in, out)):
 *   MOE_EXPERT_LINEAR   : x @ W_in[e]                            (fp32 only)  [MLG Inputs]
 *   MOE_EXPERT_RELU_MLP : relu(x @ W_in[e]) @ W_out[e]           (bf16 only)  [PFD The code; EB]
 *   MOE_EXPERT_SWIGLU   : (silu(x @ W_in[e]) * (x @ W_up[e])) @ W_out[e]
 *                         silu(z) = z / (1 + exp(-z))            (bf16 only)  [MLG Background; PFD]
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer unless stated otherwise.
 *     The caller allocates and owns every buffer, the workspace included;
 *     the library never allocates or frees device memory and keeps no state
 *     between calls other than a per-device cache of the SM count.
 *   - All calls are asynchronous on `stream` (NULL = legacy default stream)
 *     and never synchronise the host, except moe_device_status.
 *   - Host-side argument checks run before any CUDA call and return
 *     MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE.
 *     A failed kernel launch returns MOE_ERR_CUDA.  Range errors found on the
 *     device (an expert index outside [0, E), inconsistent offsets, a
 *     pipeline wait that exceeded its time limit) are written to an error
 *     word in the workspace and reported by moe_device_status.
 *   - Row-major layouts; rows of x, x_perm, y_perm and output are contiguous.
 *   - x, x_perm, y_perm, output, W_in, W_up and W_out start on a 16-byte
 *     boundary (they are moved with 16-byte vectors and TMA); a misaligned
 *     one is rejected with MOE_ERR_INVALID_ARG.
 *   - bf16 tensors are IEEE bfloat16 (upper half of an fp32).
 *   - Inputs must be finite; results for NaN or Inf inputs are undefined.
 *   - T = 0 is valid: nothing is routed, prob_mean, f and aux_loss are 0.
 *
 * Limits (MOE_ERR_UNSUPPORTED otherwise): 1 <= E <= 256; 1 <= top_k <=
 * min(E, 8); 0 <= T and T * top_k < 2^31; d, d_hidden, d_out >= 8 and
 * multiples of 8; expert_kind/act_dtype one of the three pairs above.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t. */
typedef struct CUstream_st* moe_stream_t;

enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, bad size, top_k out of range    */
  MOE_ERR_UNSUPPORTED = 2,   /* valid for the method, not built here           */
  MOE_ERR_WORKSPACE = 3,     /* workspace null, too small or misaligned        */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed    */
  MOE_ERR_DEVICE_CHECK = 5   /* a kernel flagged a range or timeout error      */
};

enum { MOE_EXPERT_LINEAR = 0, MOE_EXPERT_RELU_MLP = 1, MOE_EXPERT_SWIGLU = 2 };
enum { MOE_F32 = 0, MOE_BF16 = 1 };

/* Shapes and options of one layer call.  [MLG Inputs] x (T, d),
 * W_router (d, E), expert weights (E, ...), top_k; [MLG Follow-up]
 * capacity_factor. */
typedef struct {
  int32_t T;               /* tokens in the batch                             */
  int32_t d;               /* model width: router and expert input            */
  int32_t d_hidden;        /* expert hidden width (ReLU MLP, SwiGLU)          */
  int32_t d_out;           /* expert output width                             */
  int32_t E;               /* experts                                         */
  int32_t top_k;           /* experts per token                               */
  int32_t expert_kind;     /* MOE_EXPERT_*                                    */
  int32_t act_dtype;       /* MOE_F32 or MOE_BF16: x, expert weights, outputs */
  float capacity_factor;   /* <= 0: no capacity limit                         */
} moe_config_t;

/* Bytes of device workspace that every entry point below needs for `cfg`
 * (the same figure for all of them; it is sized for moe_forward, which keeps
 * every intermediate there).  Returns 0 if `cfg` is null or invalid. */
size_t moe_workspace_size(const moe_config_t* cfg);

/* Clears the workspace's error word (first 256 bytes), asynchronously on
 * `stream`.  Call once after allocating a workspace, before its first use.
 * ws must be 256-byte aligned. */
int moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream);

/* Synchronises `stream`, then copies the workspace's device error word to
 * *code_out (0 = no device-side error since the last clear) and clears it.
 * The word holds the first error recorded: 1 an expert index outside [0, E);
 * 2 offsets that are not a partition of the row buffer; 3 a gathered row
 * index (perm_token) outside [0, T), or a slot's grouped row (dest) at or
 * beyond T * top_k in the fused combine; 4 a sharded dispatch whose exchange
 * record for this rank is not its own, or whose records' token counts do
 * not add up to T_global; 20 moe_check_wait_timeout's
 * intended timeout; 16-19 a pipeline wait that ran out of
 * time (TMA producer, MMA issuer, epilogue, teardown drain).
 * Returns MOE_ERR_DEVICE_CHECK if the word was non-zero, MOE_OK otherwise. */
int moe_device_status(void* ws, size_t ws_bytes, int32_t* code_out, moe_stream_t stream);

/* Router: logits, softmax, top-k and renormalised gates.
 * [MLG Algorithm 1-2; PFD The code, `router`]
 *   x            (T, d) act_dtype
 *   W_router     (d, E) fp32
 *   logit_bias   (E) fp32 or NULL: added to every token's logits
 *   noise        (T, E) fp32 or NULL: added after the bias (noisy gating;
 *                the caller draws it)
 *   expert_indices (T, top_k) int32 out: by descending logit, lower index first on ties
 *   gates        (T, top_k) fp32 out, aligned with expert_indices
 *   prob_mean    (E) fp32 out: P_e = mean over tokens of softmax(logits)[:, e]
 *   logits_out   (T, E) fp32 out or NULL: the fp32 logits the top-k decided on
 * The logits are fp32: the dot product is accumulated in fp32, then the
 * bias and then the noise are each added in fp32.  With bf16 x and E <= 64
 * the dot product runs on the tensor cores: W_router is split exactly into
 * three bf16 terms (hi + mid + lo), so every product x_i * W_part is exact in
 * fp32; the tensor core's fp32 accumulator sums one 64-wide block of d at a
 * time and the blocks are added in round-to-nearest fp32.  The workspace
 * holds the split (3 * EP * d bf16, EP = E rounded up to 16, 32 or 64).
 * Otherwise the fp32 pipes compute it. */
int moe_route(const moe_config_t* cfg, const void* x, const float* W_router,
              const float* logit_bias, const float* noise,
              int32_t* expert_indices, float* gates, float* prob_mean, float* logits_out,
              void* ws, size_t ws_bytes, moe_stream_t stream);

/* The noisy gate's noise, drawn on the device: noise_out[t, e] =
 * z(token_base + t, e) * softplus((x @ W_noise)[t, e]), to pass as moe_route's
 * or moe_forward's `noise`.  [PFD The code, `router`: noise added to the
 * logits; the noisy top-k gate: a standard normal scaled by
 * softplus(x @ W_noise)]
 *   x          (T, d) bf16 (this call supports bf16 activations, E <= 64)
 *   W_noise    (d, E) fp32 row-major
 *   seed, offset  the draws are Philox4x64-10 (Salmon et al., SC 2011) of the
 *              counter (token, e, offset, 0) under the key (seed, 0); two
 *              64-bit words give u = ((w >> 11) + 1/2) / 2^53 in (0, 1) and
 *              z = sqrt(-2 ln u0) cos(2 pi u1) (Box-Muller, fp64).  Change
 *              `offset` (e.g. a step counter) for fresh noise; the same
 *              (seed, offset) always gives the same noise.
 *   token_base index of this call's first token in the whole batch (0 for a
 *              single batch; a rank's first token for a sharded one), so a
 *              sharded batch draws exactly the single batch's noise.
 *   noise_out  (T, E) fp32 out.
 * The noise logits are fp32 (the tensor-core contraction of moe_route, with
 * W_noise split exactly into three bf16 terms); softplus and the product
 * are fp64, rounded once to fp32.  Uses the workspace's split-weight area
 * (so not concurrently with moe_route on the same workspace). */
int moe_gate_noise(const moe_config_t* cfg, const void* x, const float* W_noise, uint64_t seed,
                   uint64_t offset, int64_t token_base, float* noise_out, void* ws,
                   size_t ws_bytes, moe_stream_t stream);

/* moe_route with the noisy gate's noise made inside the router: logits =
 * x @ W_router (+ logit_bias) + z(token_base + t, e) * softplus((x @ W_noise)
 * [t, e]), the noise exactly as moe_gate_noise draws it (same Philox stream,
 * same fp32 noise logits, same fp64 softplus and product), so the results
 * equal moe_gate_noise followed by moe_route bit for bit -- but the noise
 * logits come out of the router's own tensor-core contraction (W_noise rides
 * as three more bf16 terms of the B operand) and the (T, E) noise never
 * reaches memory unless noise_out asks for it.  [PFD The code, `router`:
 * the noisy top-k gate]
 *   bf16 activations and E <= 64 only (MOE_ERR_UNSUPPORTED otherwise: fp32
 *   tokens and wider gates take moe_gate_noise's noise into moe_route, or
 *   noise of their own).
 *   W_noise (d, E) fp32; seed, offset, token_base as in moe_gate_noise;
 *   noise_out (T, E) fp32 out or NULL; the other arguments as in moe_route. */
int moe_route_noisy(const moe_config_t* cfg, const void* x, const float* W_router,
                    const float* logit_bias, const float* W_noise, uint64_t seed, uint64_t offset,
                    int64_t token_base, int32_t* expert_indices, float* gates, float* prob_mean,
                    float* logits_out, float* noise_out, void* ws, size_t ws_bytes,
                    moe_stream_t stream);

/* moe_route without a workspace.  The pages have no counterpart: this entry
 * point exists for callers that cannot allocate device memory -- for
 * example a plugin running inside a host program whose memory pool owns the
 * whole GPU and hands out no scratch, or a service that forbids allocation
 * once it is serving.  Arguments, outputs and results are those of
 * moe_route; the caller still passes every input and output buffer.
 *   Scratch: the per-CTA column sums of the probabilities go to one fixed
 *   array inside the library, 65536 floats (256 KiB), which every GPU that
 *   loads the library keeps until the process exits.  A call needs
 *   ceil(T / 32) * E floats of it; larger calls return MOE_ERR_UNSUPPORTED
 *   (use moe_route with a workspace instead).  The array is overwritten in
 *   full by each call before it is read, so nothing needs clearing.
 *   Sharing: every call on a device uses the same array and it keeps the
 *   last call's contents, so calls whose kernels overlap on the GPU (on
 *   different streams, or from different host threads without ordering)
 *   race on it; order such calls on one stream.
 *   Set-up: the first call on each device looks up the array's device
 *   address (with that device current) and caches it with the id of the
 *   device's current context; make that first call before any stream
 *   capture.  The cache does not outlive the context: after cudaDeviceReset
 *   (or any new context on the device) the module is loaded again, the
 *   array may move, and the next call looks the address up afresh -- so
 *   that call, too, should come before any capture.  No call allocates or
 *   frees memory.
 *   Arithmetic: this entry point always computes the logits on the fp32
 *   pipes (it has no room for moe_route's split copy of W_router), so its
 *   logits may differ from moe_route's in the last bits; both are fp32 dot
 *   products of the same inputs. */
int moe_route_noalloc(const moe_config_t* cfg, const void* x, const float* W_router,
                      const float* logit_bias, const float* noise,
                      int32_t* expert_indices, float* gates, float* prob_mean, float* logits_out,
                      moe_stream_t stream);

/* Dispatch: per-expert histogram, positions in token order, capacity, the
 * grouped (expert-major) row layout, the load-balancing loss, and the
 * gather of token rows into that layout.
 * [MLG Algorithm 3-4, Follow-up; PFD The code, `moe_forward`, Switch]
 *   x            (T, d) act_dtype
 *   expert_indices (T, top_k) int32, each in [0, E)
 *   prob_mean    (E) fp32: P_e (from moe_route)
 *   counts       (E) int32 out: slots routed to e, before capacity
 *   offsets      (E+1) int32 out: exclusive scan of kept = min(counts, cap);
 *                expert e owns grouped rows [offsets[e], offsets[e+1])
 *   dest         (T, top_k) int32 out: grouped row of slot (t, j), or -1 if dropped
 *   perm_token   (T * top_k) int32 out: token of each grouped row; entries
 *                at and beyond offsets[E] are left untouched
 *   drop_mask    (T, top_k) uint8 out: 1 where the slot was dropped
 *   f            (E) fp32 out: counts / (T * top_k)
 *   aux_loss     (1) fp32 out: E * sum_e f_e * P_e (f before capacity)
 *   x_perm       (T * top_k, d) act_dtype out: x_perm[dest[t,j]] = x[t]; or
 *                NULL: the rows are not copied (moe_expert_ffn_gather reads
 *                them from x through perm_token instead)
 * Bit-exact and deterministic: no floating-point atomics, no order that
 * depends on scheduling. */
int moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* expert_indices,
                 const float* prob_mean, int32_t* counts, int32_t* offsets, int32_t* dest,
                 int32_t* perm_token, uint8_t* drop_mask, float* f, float* aux_loss,
                 void* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream);

/* A batch split over `world` ranks (GPUs), each holding a contiguous block of
 * its tokens, in rank order: rank 0 the first cfg->T tokens, and so on.  The
 * layer's two couplings across tokens are then global: P_e and f_e (hence
 * aux) are means over the whole batch, and a slot's position on its expert
 * counts the earlier ranks' slots first, so the capacity keeps and drops
 * exactly the slots the single-batch layer would.  [MLG Algorithm 3-4 and
 * Follow-up: positions in token order, capacity from the batch size; the
 * pages do not split a batch, so this is the single-batch rule restated]
 * Each rank contributes one exchange record of 2E+1 int32 (moe_shard_record):
 * its E slot counts per expert, its E probability means P_e over its own
 * tokens (fp32 bit patterns) and its token count.  The caller gathers every
 * rank's record in rank order (an all-gather of 2E+1 ints per rank: NCCL or
 * any collective; the library keeps to one GPU) and passes them here:
 *   rank, world   this rank and the number of ranks (0 <= rank < world)
 *   T_global      tokens of the whole batch (every rank's cfg->T summed)
 *   records       (world, 2E+1) int32 device: every rank's record in rank order
 * From the records moe_dispatch_shard takes the earlier ranks' slots per
 * expert, the batch's f_e, and the batch's P_e = (sum over ranks r in order
 * of P_e(r) * T(r)) / T_global in fp64, rounded to fp32. */
typedef struct {
  int32_t rank;
  int32_t world;
  int32_t T_global;
  const int32_t* records;
} moe_shard_t;

/* Per-expert slot counts of expert_indices (T, top_k) into counts (E) int32
 * (before any capacity). */
int moe_dispatch_count(const moe_config_t* cfg, const int32_t* expert_indices, int32_t* counts,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* This rank's exchange record (see moe_shard_t) into record (2E+1) int32:
 * the slot counts of expert_indices (T, top_k) per expert, the fp32 bits of
 * prob_mean (E) (moe_route's P over this rank's tokens) and cfg->T. */
int moe_shard_record(const moe_config_t* cfg, const int32_t* expert_indices,
                     const float* prob_mean, int32_t* record, void* ws, size_t ws_bytes,
                     moe_stream_t stream);

/* moe_dispatch for one rank of a sharded batch (see moe_shard_t).  Outputs
 * as moe_dispatch, with: counts = this rank's slots per expert; offsets,
 * dest, perm_token and x_perm describe this rank's kept rows only (its own
 * grouped layout); drop_mask holds the whole batch's keep decision for this
 * rank's slots (capacity = ceil(((capacity_factor * T_global) * top_k) / E),
 * positions offset by earlier ranks' slots); f and aux_loss are the whole
 * batch's and the same on every rank.  prob_mean is not read (may be NULL):
 * the batch's P comes from the records.  A rank whose record's counts differ
 * from its own, or records whose token counts do not add up to T_global,
 * record device error 4. */
int moe_dispatch_shard(const moe_config_t* cfg, const moe_shard_t* shard, const void* x,
                       const int32_t* expert_indices, const float* prob_mean, int32_t* counts,
                       int32_t* offsets, int32_t* dest, int32_t* perm_token, uint8_t* drop_mask,
                       float* f, float* aux_loss, void* x_perm, void* ws, size_t ws_bytes,
                       moe_stream_t stream);

/* Experts on their grouped rows: rows [offsets[e], offsets[e+1]) of x_perm
 * go through expert e and land in the same rows of y_perm.
 * [MLG Algorithm 3, Constraints: each expert runs only on its routed tokens]
 *   x_perm (R_max, d) act_dtype with R_max = T * top_k; offsets (E+1) int32
 *   with 0 = offsets[0] <= ... <= offsets[E] <= R_max.
 *   LINEAR (fp32):   W_in (E, d, d_out); W_up, W_out NULL.
 *   RELU_MLP (bf16): W_in (E, d, d_hidden), W_out (E, d_hidden, d_out); W_up NULL.
 *   SWIGLU (bf16):   W_in = W_gate (E, d, d_hidden), W_up (E, d, d_hidden),
 *                    W_out = W_down (E, d_hidden, d_out).
 *   y_perm (R_max, d_out) fp32 out (for every expert kind): each expert's
 *   output, unrounded; rows at and beyond offsets[E] are left untouched.
 * bf16 experts run on tcgen05 tensor cores with fp32 accumulation in tensor
 * memory; the hidden activation is rounded to bf16 between the two
 * projections (it is the second projection's tensor-core operand); the
 * output stays fp32 until the combine rounds the layer output once.
 * The fp32 linear expert runs in fp32 FMA. */
int moe_expert_ffn(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                   const void* W_in, const void* W_up, const void* W_out, void* y_perm,
                   void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_expert_ffn with the permute fused into the first projection: grouped
 * row r is token row x[perm_token[r]], read in place by TMA row gathers, so
 * no x_perm is ever written.  [MLG Algorithm 3: each expert gathers its own
 * tokens; the grouped layout is moe_dispatch's]
 *   x           (T, d) act_dtype, the layer input
 *   perm_token  (T * top_k) int32 from moe_dispatch: rows [0, offsets[E])
 *               must hold token indices in [0, T); an index outside it is
 *               recorded on the error word (code 3) and row 0 is used
 *   offsets, W_in, W_up, W_out, y_perm: as for moe_expert_ffn, with the same
 *               results (every row is bit-identical to moe_expert_ffn on the
 *               x_perm that moe_dispatch would have gathered).
 * Use: no (T * top_k, d) x_perm buffer is needed.  Cost: the row gathers
 * (four 128-byte rows per TMA instruction) are repeated for every output
 * column block of the first projection; on B200 at the Mixtral shape the
 * experts took 10.2 ms this way against 4.8 ms on a materialised x_perm
 * (whose copy costs about 38 us), so moe_forward gathers into x_perm. */
int moe_expert_ffn_gather(const moe_config_t* cfg, const void* x, const int32_t* perm_token,
                          const int32_t* offsets, const void* W_in, const void* W_up,
                          const void* W_out, void* y_perm, void* ws, size_t ws_bytes,
                          moe_stream_t stream);

/* The experts and the combine in one call: output as moe_combine would
 * write it from moe_expert_ffn's rows.  [MLG Algorithm 3; PFD Switch: top-1,
 * a dropped token outputs 0]  With bf16 experts the combine is the down
 * projection's epilogue and no combine kernel runs:
 *   top_k = 1: each kept grouped row r writes gates[t] * row into output row
 *     t = perm_token[r] (the same fp32 product and one rounding as
 *     moe_combine, so the same bits); no y_perm is written.
 *   top_k > 1: each kept row is also written, fp32, to the workspace's
 *     y_perm; after a row has written an output column block it counts
 *     itself on its token's counter for that block (acquire-release atomic
 *     add), and the row that completes the token's kept slots sums the
 *     token's rows for the block in increasing j with moe_combine's fp32
 *     chain and rounds once: the bits of moe_combine, whatever order the
 *     tiles finish in.  The up projection zeroes the counters first.
 * Tokens with every slot dropped get a zero row.  fp32 linear experts run
 * moe_expert_ffn into the workspace's y_perm, then the combine kernel.
 *   x_perm, offsets, perm_token, dest, gates: moe_dispatch's (and
 *   moe_route's) outputs, mutually consistent (dest[t, j] >= 0 is the
 *   grouped row whose perm_token is t); a perm_token outside [0, T) or a
 *   dest at or beyond T * top_k is recorded on the error word (code 3) and
 *   skipped.  W_in, W_up, W_out as in moe_expert_ffn;
 *   output (T, d_out) act_dtype out. */
int moe_expert_ffn_combine(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                           const int32_t* perm_token, const int32_t* dest, const float* gates,
                           const void* W_in, const void* W_up, const void* W_out, void* output,
                           void* ws, size_t ws_bytes, moe_stream_t stream);

/* Which form moe_forward uses for the experts and the combine: *fused = 1
 * when it is moe_expert_ffn_combine's combine in the down projection's
 * epilogue, 0 when it is moe_expert_ffn then moe_combine (fp32 linear
 * experts always; bf16 top_k > 1 unless the hidden width is at least 4096
 * and there are at least 1024 * E grouped rows, where the epilogue's extra
 * reads hide behind long tiles: measured on B200, 0.994x the two-call time
 * at the Mixtral shape, 1.18x at E = 64, top_k = 6, d_hidden = 1408).
 * Host-only: no CUDA call.  Returns MOE_OK, or the config check's status. */
int moe_forward_combine_fused(const moe_config_t* cfg, int32_t* fused);

/* Combine: output[t] = sum over j = 0..top_k-1 with dest[t,j] >= 0 of
 * gates[t,j] * y_perm[dest[t,j]], accumulated in fp32 in increasing j,
 * rounded once to act_dtype; a token with every slot dropped gets 0.
 * No atomics.  [MLG Algorithm 3; PFD Switch]
 *   y_perm (rows, d_out) fp32 (moe_expert_ffn's output); dest, gates
 *   (T, top_k); output (T, d_out) act_dtype. */
int moe_combine(const moe_config_t* cfg, const void* y_perm, const int32_t* dest,
                const float* gates, void* output, moe_stream_t stream);

/* The whole layer in one call: route, dispatch, experts, combine.
 * Returns the [MLG Expected Return Format] quantities:
 *   output (T, d_out) act_dtype, expert_indices (T, top_k) int32,
 *   gates (T, top_k) fp32, aux_loss (1) fp32 -- all device pointers;
 *   counts (E) int32 and drop_mask (T, top_k) uint8 are optional (NULL).
 * Inputs as in moe_route and moe_expert_ffn.  Intermediates live in ws.
 * The experts and the combine run as moe_expert_ffn_combine, or as
 * moe_expert_ffn into the workspace's y_perm followed by moe_combine, as
 * moe_forward_combine_fused reports for cfg; the output bits are the same. */
int moe_forward(const moe_config_t* cfg, const void* x, const float* W_router,
                const float* logit_bias, const float* noise,
                const void* W_in, const void* W_up, const void* W_out,
                void* output, int32_t* expert_indices, float* gates, float* aux_loss,
                int32_t* counts, uint8_t* drop_mask,
                void* ws, size_t ws_bytes, moe_stream_t stream);

/* Backward of the routing half (combine and router), for training.  The
 * pages print no backward; these are the derivatives of the forward above.
 * [MLG Algorithm 2-4; PFD The code, `switch_balance_loss`: f is a count and
 * carries no gradient, P_e does]
 *
 * moe_combine_backward: from dy = dLoss/d output (T, d_out) act_dtype:
 *   dy_perm (T*top_k, d_out) fp32 out: row dest[t,j] = gates[t,j] * dy[t]
 *           (the gradient into the experts' outputs; other rows untouched)
 *   dgates  (T, top_k) fp32 out: <dy[t], y_perm[dest[t,j]]>, 0 if dropped
 *   y_perm and dest, gates as in the forward (y_perm fp32, moe_expert_ffn's).
 * Fixed orders: per token, the columns in order per lane, then a fixed
 * butterfly over the warp.  No workspace. */
int moe_combine_backward(const moe_config_t* cfg, const void* dy, const void* y_perm,
                         const int32_t* dest, const float* gates, float* dy_perm, float* dgates,
                         moe_stream_t stream);

/* moe_route_backward: gradients of the gates and of aux_loss back to the
 * router's inputs.  With p = softmax(logits) per token and g the gates:
 *   dL[t,m] = g_m (dg_m - sum_j g_j dg_j) for each chosen m (the top-k
 *             choice itself has no gradient), plus
 *             p_te (a_e - sum_e' p_te' a_e'),  a_e = daux * E * f_e / T_batch
 *   dx = dL @ W_router^T, dW_router = x^T @ dL, dbias = sum_t dL.
 *   x (T, d) act_dtype; W_router (d, E) fp32; logits (T, E) fp32 (moe_route's
 *   logits_out: the logits the top-k decided on, after bias and noise);
 *   expert_indices, gates (T, top_k); f (E) fp32 (moe_dispatch's, before
 *   capacity); dgates (T, top_k) fp32 (e.g. moe_combine_backward's); daux
 *   (1) fp32 device: dLoss/d aux_loss; T_batch: tokens P_e and f_e are
 *   means over (0 = this call's T; a rank's share of a sharded batch passes
 *   the whole batch's T, and the ranks then add their dW and dbias).
 *   dx (T, d) fp32 out; dW_router (d, E) fp32 out; dbias (E) fp32 out or
 *   NULL; dlogits (T, E) fp32 out or NULL (kept in the workspace then).
 * fp32 throughout with fixed summation orders (dW and dbias: token chunks
 * in order). */
int moe_route_backward(const moe_config_t* cfg, const void* x, const float* W_router,
                       const float* logits, const int32_t* expert_indices, const float* gates,
                       const float* f, const float* dgates, const float* daux, int32_t T_batch,
                       float* dx, float* dW_router, float* dbias, float* dlogits, void* ws,
                       size_t ws_bytes, moe_stream_t stream);

/* Backward of the experts, for training.  The pages print no backward; these
 * are the derivatives of moe_expert_ffn's experts ([MLG Algorithm 3]: each
 * expert on its routed rows; [PFD The code, `expert_forward`]: the ReLU
 * expert; SwiGLU as in moe_expert_ffn; [PFD Hot shards]: an expert that
 * receives no row gets no gradient).  For the rows X of expert e, the
 * gradient dY of its outputs, A = X W_in (B = X W_up) and H the hidden
 * activation:
 *   dH = dY W_out^T
 *   ReLU:   dA = dH * [A > 0]
 *   SwiGLU: s = sigmoid(A), dA = dH * B * s (1 + A (1 - s)), dB = dH * A s
 *   dX = dA W_in^T (+ dB W_up^T);  dW_out = H^T dY, dW_in = X^T dA,
 *   dW_up = X^T dB.  Linear experts: dX = dY W_in^T, dW_in = X^T dY.
 *
 * moe_expert_backward_workspace_size: bytes of the workspace this call
 *   needs (its own, not moe_workspace_size's; 0 on a bad config).  Its
 *   first 256 bytes are an error word like the forward workspace's
 *   (moe_workspace_init / moe_device_status apply).
 * moe_expert_ffn_backward:
 *   x_perm  (T*top_k, d) act_dtype, offsets (E+1) int32: moe_dispatch's
 *           grouped rows and their expert ranges
 *   W_in, W_up, W_out as in moe_expert_ffn (W_up NULL unless SwiGLU,
 *           W_out NULL for linear experts)
 *   dy_perm (T*top_k, d_out) fp32: gradient of each kept row's expert output
 *           (moe_combine_backward's dy_perm)
 *   dx_perm (T*top_k, d) fp32 out: gradient of each kept grouped row; rows
 *           at and beyond offsets[E] untouched
 *   dW_in, dW_up, dW_out fp32 out, shaped like the weights (E, in, out);
 *           NULL where the weight is NULL; every expert's block is written
 *           (zeros for an expert without rows)
 * bf16 experts run on the tensor cores (bf16 operands, fp32 accumulation):
 * the rows are copied into a layout padded to 64 rows per expert, dY is
 * rounded to bf16, the forward's A and B are recomputed and kept in fp32,
 * dA, dB and H are rounded to bf16 between the GEMMs.  Linear experts run
 * in fp32.  Deterministic: no atomics, fixed summation orders. */
size_t moe_expert_backward_workspace_size(const moe_config_t* cfg);
int moe_expert_ffn_backward(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                            const void* W_in, const void* W_up, const void* W_out,
                            const float* dy_perm, float* dx_perm, float* dW_in, float* dW_up,
                            float* dW_out, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Training forward of the experts and the backward that uses what it kept.
 * moe_expert_ffn_train: moe_expert_ffn (same arguments and the same y_perm,
 *   bit for bit) that also writes every kept row's fp32 pre-activations, A =
 *   X W_in (and B = X W_up for SwiGLU), into bwd_ws, the workspace of
 *   moe_expert_ffn_backward (bwd_ws_bytes >= moe_expert_backward_workspace_size;
 *   the same offsets must be given to the backward).  bf16 experts only
 *   (MOE_ERR_UNSUPPORTED for linear experts, which have no pre-activations).
 * moe_expert_ffn_backward_saved: moe_expert_ffn_backward with the same
 *   arguments, taking A and B from ws (written there by
 *   moe_expert_ffn_train on the same x_perm, offsets and weights) instead
 *   of recomputing them: a quarter of the backward's tensor work less, for
 *   (R_max + 63 E) x (1 + SwiGLU) x d_hidden fp32 written by the forward.
 *   The results equal moe_expert_ffn_backward's up to the order in which the
 *   tensor cores sum A and B. */
int moe_expert_ffn_train(const moe_config_t* cfg, const void* x_perm, const int32_t* offsets,
                         const void* W_in, const void* W_up, const void* W_out, void* y_perm,
                         void* ws, size_t ws_bytes, void* bwd_ws, size_t bwd_ws_bytes,
                         moe_stream_t stream);
int moe_expert_ffn_backward_saved(const moe_config_t* cfg, const void* x_perm,
                                  const int32_t* offsets, const void* W_in, const void* W_up,
                                  const void* W_out, const float* dy_perm, float* dx_perm,
                                  float* dW_in, float* dW_up, float* dW_out, void* ws,
                                  size_t ws_bytes, moe_stream_t stream);

/* moe_permute_backward: the grouped rows' input gradients back to their
 * tokens, dx[t] = dx_add[t] + sum over kept slots j (j increasing) of
 * dx_perm[dest[t, j]] (each token's input feeds its kept rows; [MLG
 * Algorithm 3]).  dx_perm (T*top_k, d) fp32; dest (T, top_k) int32 from
 * moe_dispatch; dx_add (T, d) fp32 or NULL (e.g. moe_route_backward's dx, so
 * that dx is the whole layer's input gradient); dx (T, d) fp32 out (may be
 * dx_add).  fp32, fixed order, no workspace. */
int moe_permute_backward(const moe_config_t* cfg, const float* dx_perm, const int32_t* dest,
                         const float* dx_add, float* dx, moe_stream_t stream);

/* Self-test of the library's failure detection; the pages have no
 * counterpart.  Every pipeline wait in the library's kernels is bounded:
 * instead of hanging, a wait that does not complete in time records an
 * error code on the workspace's error word and the kernel returns, leaving
 * the CUDA context usable.  This call runs one such wait on an mbarrier that
 * nothing completes, with a limit of limit_us microseconds (1 .. 10^7), so
 * a caller (or a health check) can see the mechanism work: afterwards
 * moe_device_status reports code 20.  It faults nothing and holds the GPU
 * for about limit_us.  ws needs only its first 256 bytes (the error word). */
int moe_check_wait_timeout(void* ws, size_t ws_bytes, uint32_t limit_us, moe_stream_t stream);

/* Static text for a status code. */
const char* moe_status_string(int status);

/* Text of the most recent non-OK status returned on this host thread
 * (argument name, CUDA error string, ...).  Empty if none. */
const char* moe_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
