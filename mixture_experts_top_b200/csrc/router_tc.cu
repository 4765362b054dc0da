// router_tc.cu - the router on the tensor cores for bf16 tokens: fp32
// logits, softmax, top-k, renormalised gates and the column sums of the
// probabilities, in one kernel.
//
// What it computes is the router of router.cu:
// "Mixture-of-Experts Routing - LLM Internals" (mlgrind.dev), Algorithm 1-2:
//   logits = x @ W_router; probs = softmax(logits); indices = the k largest
//   logits by descending value, lower index first on ties; gates = softmax
//   over the chosen k logits.
// "Mixture of Experts: the Sparsely-Gated Layer" (paperfordummies.in), The
// code, `router`: an optional per-expert bias, then optional noise, are added
// to the logits before the softmax and the top-k.
//
// fp32 logits from bf16 tensor cores.  x is bf16, so every x_i is exact.
// W_router (fp32) is split exactly into three bf16 terms, W = W_hi + W_mid +
// W_lo, each taking the next 8 significant bits of the fp32 value (the
// remainders w - W_hi and (w - W_hi) - W_mid are exact in fp32).  Every
// product x_i * W_part has at most 16 significant bits and is exact in fp32,
// and tcgen05.mma (kind::f16: bf16 in, fp32 accumulate) adds them in fp32.
// The tensor core's accumulator does not round to nearest (its errors lean
// towards zero, measured on B200), so it only sums one 64-wide block of d
// (4 MMAs); the blocks' sums are added in round-to-nearest fp32 in
// registers, in block order.  The result is an fp32 dot product like the
// scalar router's, in another summation order, and the contraction is bound
// by reading x from HBM instead of by the fp32 pipes.
//
// Design (B200)
//  * A split kernel writes (W_hi, W_mid, W_lo) as one (3, EP, d) bf16 array,
//    d contiguous (a K-major operand), rows E..EP-1 zero; EP = E padded to
//    16, 32 or 64 (the MMA's N).
//  * A thread-block cluster of S CTAs (S = 1..8) owns a tile of 128 tokens;
//    CTA r of the cluster takes every S-th 64-wide block of d, from block r
//    (the cluster reads runs of S * 128 bytes of each token row).  192 threads:
//    warp 0 lane 0 issues TMA copies (x box 64 (d) x 128 (tokens) and the
//    three W boxes 64 (d) x EP, 128-byte swizzle) into a ring of stages;
//    warp 1 lane 0 issues, per 64-wide d block, 4 tcgen05.mma M128 x N x K16
//    into a fresh fp32 accumulator in tensor memory, N = 3 EP: the three W
//    boxes lie one after another in shared memory, so one MMA forms the hi,
//    mid and lo products in three column groups (two accumulators alternate
//    for EP <= 32); warps 2-5 (warp w reads TMEM lanes 32 (w mod 4) ..) add
//    each block's hi + (mid + lo) into their token's fp32 registers and
//    release the accumulator.  Out-of-range tokens and d are zero-filled by
//    TMA.
//  * Epilogue: each token's partial logits go to shared memory; after a
//    cluster barrier, the CTA of rank r finishes tokens
//    [r 128/S, (r+1) 128/S) of the tile.  All its threads add the S partial
//    logit rows in rank order through distributed shared memory, then the
//    bias and the noise (coalesced, consecutive experts on consecutive
//    threads); then a group of EP/8 lanes per token (8 experts a lane): each
//    lane sorts its 64-bit keys (order-preserving logit bits, then the
//    complemented expert index, so the lower index wins ties) once, top-k
//    takes k rounds of a group-wide maximum of the lanes' first keys, then
//    the softmax (its maximum is the first top-k logit) and the gates.  Each
//    CTA then adds its tokens' probabilities per expert in token order, and
//    rank 0 adds the S sums in rank order into the tile's row of column sums;
//    the last tile to finish reduces the rows to P in fp64.
//  * Every mbarrier wait is bounded; on expiry the error word is set, the
//    copies in flight are drained and tensor memory is freed.
#include <cooperative_groups.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace cg = cooperative_groups;

namespace moe {
namespace {

constexpr int TBM = 128;       // tokens per CTA (UMMA M)
constexpr int TBK = 64;        // d per stage: one 128-byte swizzle row of bf16
constexpr int TUK = 16;        // d per tcgen05.mma (kind::f16)
constexpr int TTHREADS = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 accumulate and finish
constexpr int kCoopBatch = 8;  // elements per thread per round of the logit pass
constexpr int kMaxTopK = 8;    // largest top_k the library accepts
constexpr int kSplitLoads = TBK * 64 / 256;  // W loads per thread of the split (E <= 64)

// kModeRoute: the router.  kModeLogits: the contraction and the rank-ordered
// sum only, written to logits_out (the noisy gate's noise logits).
// kModeNoisy: the router with the noisy gate's noise made in the kernel: the
// B operand carries W_noise's three terms after W_router's, so each token's
// noise logits come out of the same contraction, and noise = z * softplus(
// noise logit) is formed in the logit pass (the (T, E) noise never reaches
// memory unless asked for).
enum TcMode { kModeRoute = 0, kModeLogits = 1, kModeNoisy = 2 };

template <int EP, int MODE>
struct TcShape {
  static_assert(EP == 16 || EP == 32 || EP == 64, "EP is 16, 32 or 64");
  static constexpr bool NOISY = MODE == kModeNoisy;
  static constexpr int TERMS = NOISY ? 6 : 3;                    // hi, mid, lo (x2 noisy)
  static constexpr int ST = NOISY ? (EP == 16 ? 3 : 2) : (EP == 16 ? 4 : (EP == 32 ? 3 : 2));
  static constexpr int X_BYTES = TBM * TBK * 2;                  // 16 KiB
  static constexpr int W_PART = EP * TBK * 2;                    // one term's box
  static constexpr int STAGE = X_BYTES + TERMS * W_PART;
  static constexpr int LOGW = NOISY ? 2 * EP : EP;               // a token's logits (+ noise logits)
  static constexpr int LGS = LOGW + 4;                           // padded logit row (floats)
  static constexpr int PIPE = ST * STAGE;
  static constexpr int LG_BYTES = TBM * LGS * 4;
  static constexpr int MAIN = PIPE > LG_BYTES ? PIPE : LG_BYTES;
  static constexpr int AUX = 256;                                // barriers, TMEM address
  static constexpr int SMEM = 1024 + MAIN + EP * 4 + AUX;
  // B is the TERMS * EP rows of the stage (W's hi, mid, lo, then W_noise's),
  // so an accumulator is TERMS * EP columns, issued as one MMA (or two of half
  // the width where that exceeds the instruction's 256).  Up to four
  // accumulators rotate within 256 columns (the MMA runs ahead of the
  // registers' block sums by that many blocks): four at EP = 16, two at
  // EP = 32, one at EP = 64 or with the noise terms at EP > 16.
  static constexpr int N = TERMS * EP;
  static constexpr int NMMA = N <= 256 ? N : N / 2;
  static constexpr int MMAS = N / NMMA;
  static constexpr int NBUF = N > 128 ? 1 : (256 / N >= 4 ? 4 : 2);
  static constexpr int G = 1;   // 64-wide d blocks summed per accumulator before it is read
  static constexpr int FG = EP / 8;  // lanes per token in the finishing pass (8 experts each)
  static constexpr uint32_t TMEM_COLS = NBUF * N <= 32 ? 32u : NBUF * N <= 64 ? 64u
                                        : NBUF * N <= 128 ? 128u : NBUF * N <= 256 ? 256u : 512u;
  static constexpr int CTAS_PER_SM = TMEM_COLS > 256 ? 1 : 2;
  // kind::f16: D fp32 (bit 4), A bf16 (bits 7-9 = 1), B bf16 (bits 10-12 =
  // 1), A and B K-major (bits 15, 16 = 0), N >> 3 at 17, M >> 4 at 24.
  static constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) |
                                    ((uint32_t)(NMMA >> 3) << 17) | ((uint32_t)(TBM >> 4) << 24);
  static_assert(NBUF * N <= 512 && NMMA % 16 == 0 && NMMA * MMAS == N, "accumulators fit");
  static_assert((NMMA * 128) % 1024 == 0, "second MMA's B starts on an 8-row group");
  static_assert((2 * ST + 2 * NBUF + 1) * 8 + 4 <= AUX, "barriers fit");
};

// K-major operand, 128-byte swizzle: rows of 128 bytes, 8-row groups 1024
// bytes apart (stride byte offset); the leading byte offset is unused for
// this layout (16 bytes); descriptor version 1 (bit 46); swizzle mode 2.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

struct TcArgs {
  const float* bias;
  const float* noise;
  int32_t* idx;
  float* gates;
  float* logits_out;
  float* part;
  int32_t* err;
  int T, d, E, k;
  // kModeNoisy: the noise's Philox key and stream, the batch index of this
  // call's first token, and an optional (T, E) copy of the noise drawn.
  uint64_t seed, offset;
  long long token_base;
  float* noise_out;
  const double* noise_z;   // (T, E) the draws z, made before the router runs
  // kModeRoute / kModeNoisy: P_e, written by the last tile to finish, which
  // it finds with a counter that starts at 0 and is left at 0.
  float* prob_mean;
  unsigned* done;
};

// Philox4x64-10 (Salmon, Moraes, Dror and Shaw, "Parallel random numbers: as
// easy as 1, 2, 3", SC 2011): ten rounds over a 4-word counter, the key
// advanced by the two Weyl constants between rounds.
__device__ __forceinline__ void philox4x64_10(uint64_t (&x)[4], uint64_t k0, uint64_t k1) {
  constexpr uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
  constexpr uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += W0;
      k1 += W1;
    }
    const uint64_t hi0 = __umul64hi(M0, x[0]), lo0 = M0 * x[0];
    const uint64_t hi1 = __umul64hi(M1, x[2]), lo1 = M1 * x[2];
    const uint64_t y0 = hi1 ^ x[1] ^ k0, y2 = hi0 ^ x[3] ^ k1;
    x[0] = y0;
    x[1] = lo1;
    x[2] = y2;
    x[3] = lo0;
  }
}

// The noisy gate's noise of batch token t and expert e from its noise logit
// l: z * softplus(l), z the standard normal drawn from Philox4x64-10 of the
// counter (t, e, offset, 0) under the key (seed, 0): two words to u = ((w >>
// 11) + 1/2) 2^-53 and z = sqrt(-2 ln u0) cos(2 pi u1) (Box-Muller), in
// fp64; softplus(l) = max(l, 0) + log1p(exp(-|l|)) in fp64; one rounding.
__device__ __forceinline__ double gate_noise_z(uint64_t seed, uint64_t offset, long long t,
                                               int e) {
  uint64_t w[4] = {(uint64_t)t, (uint64_t)e, offset, 0ull};
  philox4x64_10(w, seed, 0ull);
  const double u0 = ((double)(w[0] >> 11) + 0.5) * 0x1.0p-53;
  const double u1 = ((double)(w[1] >> 11) + 0.5) * 0x1.0p-53;
  return sqrt(-2.0 * log(u0)) * cos(2.0 * 3.141592653589793 * u1);
}
__device__ __forceinline__ float gate_noise_from_z(double z, float l) {
  const double ld = (double)l;
  const double sp = fmax(ld, 0.0) + log1p(exp(-fabs(ld)));
  return (float)(z * sp);
}
__device__ __forceinline__ float gate_noise_value(uint64_t seed, uint64_t offset, long long t,
                                                  int e, float l) {
  return gate_noise_from_z(gate_noise_z(seed, offset, t, e), l);
}

// Sorts 8 keys into descending order: a 19-comparator, depth-6 network
// (checked on all 256 zero-one inputs, which by the zero-one principle
// covers every input).
__device__ __forceinline__ void cmpx_desc(uint64_t& a, uint64_t& b) {
  const uint64_t hi = a > b ? a : b, lo = a > b ? b : a;
  a = hi;
  b = lo;
}
__device__ __forceinline__ void sort8_desc(uint64_t (&v)[8]) {
  cmpx_desc(v[0], v[2]); cmpx_desc(v[1], v[3]); cmpx_desc(v[4], v[6]); cmpx_desc(v[5], v[7]);
  cmpx_desc(v[0], v[4]); cmpx_desc(v[1], v[5]); cmpx_desc(v[2], v[6]); cmpx_desc(v[3], v[7]);
  cmpx_desc(v[0], v[1]); cmpx_desc(v[2], v[3]); cmpx_desc(v[4], v[5]); cmpx_desc(v[6], v[7]);
  cmpx_desc(v[2], v[4]); cmpx_desc(v[3], v[5]);
  cmpx_desc(v[1], v[4]); cmpx_desc(v[3], v[6]);
  cmpx_desc(v[1], v[2]); cmpx_desc(v[3], v[4]); cmpx_desc(v[5], v[6]);
}

// (d, E) fp32 -> (3, EP, d) bf16 terms hi, mid, lo with w = hi + mid + lo.
// One block per 64 rows of d, transposed through shared memory; blockIdx.y
// = 1 splits W2 into the next three planes.
// With z_out, the blocks of blockIdx.y = 2 instead draw the noisy gate's
// z for every (token, expert) of the call (they depend on neither input).
struct NoiseDraw {
  double* z_out;          // (T, E) or nullptr
  uint64_t seed, offset;
  long long token_base;
  int T;
};

__global__ void __launch_bounds__(256)
    split_router_weights_kernel(const float* __restrict__ W1, const float* __restrict__ W2, int d,
                                int E, int EP, __nv_bfloat16* __restrict__ out_base,
                                const NoiseDraw nd) {
  pdl_wait_and_release();
  if (blockIdx.y == 2) {
    const long long n = (long long)nd.T * E;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
      const long long t = i / E;
      nd.z_out[i] = gate_noise_z(nd.seed, nd.offset, nd.token_base + t, (int)(i - t * E));
    }
    return;
  }
  if ((int)blockIdx.x * TBK >= d) return;
  __shared__ float tile[TBK][65];
  const float* __restrict__ W = blockIdx.y == 0 ? W1 : W2;
  __nv_bfloat16* __restrict__ out = out_base + (size_t)blockIdx.y * 3 * EP * d;
  const int k0 = blockIdx.x * TBK;
  // The block's 64 rows of W are contiguous: up to 16 loads per thread, all
  // issued before the first is used, so their latencies overlap.
  {
    const float* __restrict__ src = W + (size_t)k0 * E;
    const int n = min(TBK, d - k0) * E;
    float v[kSplitLoads];
#pragma unroll
    for (int j = 0; j < kSplitLoads; ++j) {
      const int i = threadIdx.x + j * 256;
      v[j] = i < n ? __ldg(src + i) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < kSplitLoads; ++j) {
      const int i = threadIdx.x + j * 256;
      if (i < TBK * E) {
        const int kk = i / E;
        tile[kk][i - kk * E] = v[j];
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < EP * TBK; i += blockDim.x) {
    const int e = i / TBK, kk = i % TBK;
    if (k0 + kk >= d) continue;
    const float w = e < E ? tile[kk][e] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = __fsub_rn(w, __bfloat162float(hi));      // exact
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = __fsub_rn(r1, __bfloat162float(mid));    // exact, <= 8 bits
    const size_t o = (size_t)e * d + k0 + kk;
    out[o] = hi;
    out[(size_t)EP * d + o] = mid;
    out[(size_t)2 * EP * d + o] = __float2bfloat16_rn(r2);
  }
}

template <int EP, int MODE>
__global__ void __launch_bounds__(TTHREADS, TcShape<EP, MODE>::CTAS_PER_SM)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const TcArgs a) {
  using S = TcShape<EP, MODE>;
  constexpr bool LOGITS_ONLY = MODE == kModeLogits;
  constexpr bool NOISY = MODE == kModeNoisy;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* lg = reinterpret_cast<float*>(smem);                  // after the main loop
  float* csum = reinterpret_cast<float*>(smem + S::MAIN);      // EP floats
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + S::MAIN + EP * 4);
  uint64_t* empty_bar = full_bar + S::ST;
  uint64_t* tfull_bar = empty_bar + S::ST;   // [NBUF] accumulator written
  uint64_t* tempty_bar = tfull_bar + S::NBUF;  // [NBUF] accumulator read
  uint64_t* drain_bar = tempty_bar + S::NBUF;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain_bar + 1);

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int nsplit = (int)cluster.num_blocks();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = a.T, E = a.E;
  const int tile = blockIdx.x / nsplit;
  const int t_base = tile * TBM;
  const int total_chunks = (a.d + TBK - 1) / TBK;
  // CTA r takes the 64-wide d blocks r, r + S, r + 2S, ...: the S CTAs of a
  // tile read neighbouring 128-byte pieces of the same token rows at about
  // the same time, so HBM sees runs of S * 128 bytes instead of scattered
  // 128-byte reads.
  const int nchunks = rank < total_chunks ? (total_chunks - rank + nsplit - 1) / nsplit : 0;

  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmX);
    tma_prefetch_map(&tmW);
  } else if (warp == 1) {
    tmem_alloc(tmem_holder, S::TMEM_COLS);
    tmem_relinquish();
  } else if (warp == 2 && lane == 0) {
    for (int s = 0; s < S::ST; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < S::NBUF; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 128);
    }
    mbar_init(drain_bar, 1);
    fence_mbar_init();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_holder;
  // The set-up above reads no input, so it overlaps the previous kernel's
  // tail; every read of x, W and the outputs' buffers comes after this.
  pdl_wait_and_release();

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- TMA producer
    int stage = 0;
    uint32_t phase = 0, issued = 0, last_phase = 0;
    for (int c = 0; c < nchunks; ++c) {
      if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) {
        report_error(a.err, kDevTimeoutProducer);
        break;
      }
      uint8_t* sx = smem + stage * S::STAGE;
      const int k0 = (rank + c * nsplit) * TBK;
      mbar_arrive_expect_tx(&full_bar[stage], S::STAGE);
      tma_load_2d(sx, &tmX, &full_bar[stage], k0, t_base);
      tma_load_3d(sx + S::X_BYTES, &tmW, &full_bar[stage], k0, 0, 0);
      issued |= 1u << stage;
      last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
      if (++stage == S::ST) {
        stage = 0;
        phase ^= 1u;
      }
    }
    for (int s = 0; s < S::ST; ++s)
      if ((issued >> s) & 1u)
        if (!mbar_wait(&full_bar[s], (last_phase >> s) & 1u)) report_error(a.err, kDevTimeoutDrain);
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    for (int c = 0; c < nchunks; ++c) {
      const int gi = c / S::G, b = gi % S::NBUF;
      const bool first = (c % S::G) == 0;
      if ((first && !mbar_wait(&tempty_bar[b], ((uint32_t)(gi / S::NBUF) & 1u) ^ 1u)) ||
          !mbar_wait(&full_bar[stage], phase)) {
        report_error(a.err, kDevTimeoutMma);
        break;
      }
      tc_fence_after_sync();
      const uint32_t sx = smem_u32(smem + stage * S::STAGE);
      const uint32_t sw = sx + S::X_BYTES;
      const uint32_t acc = tmem + (uint32_t)(b * S::N);
#pragma unroll
      for (int kk = 0; kk < TBK / TUK; ++kk)
#pragma unroll
        for (int m = 0; m < S::MMAS; ++m)
          umma_bf16_ss(acc + (uint32_t)(m * S::NMMA), desc_kmajor_sw128(sx + kk * TUK * 2),
                       desc_kmajor_sw128(sw + m * S::NMMA * 128 + kk * TUK * 2), S::IDESC,
                       (!first || kk != 0) ? 1u : 0u);
      umma_commit(&empty_bar[stage]);   // frees the stage once these MMAs finish
      if ((c % S::G) == S::G - 1 || c == nchunks - 1)
        umma_commit(&tfull_bar[b]);     // this group's sums are ready
      if (++stage == S::ST) {
        stage = 0;
        phase ^= 1u;
      }
    }
    umma_commit(drain_bar);  // every MMA issued above completes before TMEM is freed
    if (!mbar_wait(drain_bar, 0)) report_error(a.err, kDevTimeoutDrain);
  } else if (warp >= 2) {
    // ------------------------------- per-block sums -> fp32 registers -> smem
    const int q = warp & 3;                 // TMEM lanes 32q .. 32q + 31
    float acc[EP];
    float nacc[NOISY ? EP : 1];
#pragma unroll
    for (int e = 0; e < EP; ++e) acc[e] = 0.f;
#pragma unroll
    for (int e = 0; e < (NOISY ? EP : 1); ++e) nacc[e] = 0.f;
    const int ngroups = (nchunks + S::G - 1) / S::G;
    for (int gi = 0; gi < ngroups; ++gi) {
      const int b = gi % S::NBUF;
      const bool ready = mbar_wait(&tfull_bar[b], (uint32_t)(gi / S::NBUF) & 1u);
      if (!__all_sync(0xffffffffu, ready)) {
        if (lane == 0) report_error(a.err, kDevTimeoutEpilogue);
        break;
      }
      tc_fence_after_sync();
      // Columns [p EP, (p+1) EP) of the accumulator hold term p's block sums;
      // the block adds hi + (mid + lo) to the running fp32 logits.
      const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * S::N);
#pragma unroll
      for (int c0 = 0; c0 < EP; c0 += 16) {
        uint32_t hi[16], mid[16], lo[16];
        tmem_ld_32x32b_x16(taddr + (uint32_t)c0, hi);
        tmem_ld_32x32b_x16(taddr + (uint32_t)(EP + c0), mid);
        tmem_ld_32x32b_x16(taddr + (uint32_t)(2 * EP + c0), lo);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          acc[c0 + j] += __uint_as_float(hi[j]) + (__uint_as_float(mid[j]) + __uint_as_float(lo[j]));
        if (NOISY) {
          // columns [3 EP, 6 EP): W_noise's terms, summed the same way
          tmem_ld_32x32b_x16(taddr + (uint32_t)(3 * EP + c0), hi);
          tmem_ld_32x32b_x16(taddr + (uint32_t)(4 * EP + c0), mid);
          tmem_ld_32x32b_x16(taddr + (uint32_t)(5 * EP + c0), lo);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            nacc[(c0 + j) % (NOISY ? EP : 1)] +=
                __uint_as_float(hi[j]) + (__uint_as_float(mid[j]) + __uint_as_float(lo[j]));
        }
      }
      tc_fence_before_sync();
      mbar_arrive(&tempty_bar[b]);
    }
    float* my = lg + (q * 32 + lane) * S::LGS;
#pragma unroll
    for (int e = 0; e < EP; e += 4)
      *reinterpret_cast<float4*>(my + e) = make_float4(acc[e], acc[e + 1], acc[e + 2], acc[e + 3]);
    if (NOISY) {
#pragma unroll
      for (int e = 0; e < (NOISY ? EP : 1); e += 4)
        *reinterpret_cast<float4*>(my + EP + e) =
            make_float4(nacc[e], nacc[(e + 1) % (NOISY ? EP : 1)], nacc[(e + 2) % (NOISY ? EP : 1)],
                        nacc[(e + 3) % (NOISY ? EP : 1)]);
    }
  }
  __syncwarp();
  cluster.sync();  // every CTA's partial logits are complete and visible

  // --------------------------------------- the tile's logits, all threads
  // CTA r finishes tokens [r0, r0 + rpc) of the tile.  Their logits are the
  // partial rows of the S CTAs added in rank order (read through distributed
  // shared memory, consecutive experts on consecutive threads), then the
  // bias and the noise, each in fp32; they overwrite this CTA's own partial
  // rows, which no other CTA reads.  Each thread takes kCoopBatch elements
  // at a time and issues all their loads before using any, so the load
  // latencies overlap.
  const int rpc = TBM / nsplit;
  const int r0 = rank * rpc;
  {
    const int n = rpc * EP;
    for (int base = threadIdx.x; base < n; base += TTHREADS * kCoopBatch) {
      float acc[kCoopBatch], bv[kCoopBatch], nv[kCoopBatch], nl[kCoopBatch];
#pragma unroll
      for (int u = 0; u < kCoopBatch; ++u) {
        const int i = base + u * TTHREADS;
        acc[u] = 0.f;
        bv[u] = 0.f;
        nv[u] = 0.f;
        nl[u] = 0.f;
        const int r = r0 + i / EP, e = i % EP, t = t_base + r;
        if (i < n && e < E && t < T) {
          if (a.bias != nullptr) bv[u] = a.bias[e];
          if (!NOISY && a.noise != nullptr) nv[u] = a.noise[(size_t)t * E + e];
        }
      }
      for (int sp = 0; sp < nsplit; ++sp) {
        const float* src = cluster.map_shared_rank(lg, sp);
        float pv[kCoopBatch], pn[kCoopBatch];
#pragma unroll
        for (int u = 0; u < kCoopBatch; ++u) {
          const int i = base + u * TTHREADS;
          pv[u] = i < n ? src[(r0 + i / EP) * S::LGS + i % EP] : 0.f;
          pn[u] = (NOISY && i < n) ? src[(r0 + i / EP) * S::LGS + EP + i % EP] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kCoopBatch; ++u) {
          acc[u] += pv[u];
          nl[u] += pn[u];
        }
      }
#pragma unroll
      for (int u = 0; u < kCoopBatch; ++u) {
        const int i = base + u * TTHREADS;
        if (i < n) {
          const int r = r0 + i / EP, e = i % EP, t = t_base + r;
          float v = acc[u];
          if (e < E && t < T) {
            if (NOISY) {
              // the noise of this token and expert from its noise logit and
              // its draw (drawn ahead by the weight-split launch)
              nv[u] = gate_noise_from_z(__ldcg(a.noise_z + (size_t)t * E + e), nl[u]);
              if (a.noise_out != nullptr) a.noise_out[(size_t)t * E + e] = nv[u];
            }
            if (a.bias != nullptr) v = __fadd_rn(v, bv[u]);
            if (NOISY || a.noise != nullptr) v = __fadd_rn(v, nv[u]);
            if (a.logits_out != nullptr) a.logits_out[(size_t)t * E + e] = v;
          }
          lg[r * S::LGS + e] = v;
        }
      }
    }
  }
  __syncthreads();

  if (LOGITS_ONLY) goto teardown;
  // ------------------------------ finishing, a group of G lanes per token
  // Each lane of a group holds 8 consecutive experts' logits as 64-bit keys
  // (order-preserving logit bits, then the complemented expert index, so the
  // lower index wins ties; -0 and +0 are one key; absent experts are 0),
  // sorted once in descending order by a 19-comparator network.  Top-k: k
  // rounds of a group-wide maximum of the lanes' first keys; the lane that
  // held the winner drops it.  Softmax: the maximum is the first top-k
  // logit; the exponentials are summed per lane, then over the group, and
  // scaled by the sum's reciprocal.  The probabilities overwrite the token's
  // logit row, and the group's first lane writes indices and gates.
  {
    constexpr int G = S::FG;                         // lanes per token
    const int lane_in = lane & (G - 1);
    const uint32_t gmask = (G == 32) ? 0xffffffffu
                                     : (((1u << G) - 1u) << (lane & ~(G - 1)));
    const int group = (int)threadIdx.x / G;
    const int k = a.k;
    for (int rr = group; rr < rpc; rr += TTHREADS / G) {
      const int r = r0 + rr;
      const int t = t_base + r;
      if (t >= T) break;                             // later rows are past T too
      float* row = lg + r * S::LGS + lane_in * 8;
      float L[8];
      {
        const float4 v0 = *reinterpret_cast<const float4*>(row);
        const float4 v1 = *reinterpret_cast<const float4*>(row + 4);
        L[0] = v0.x; L[1] = v0.y; L[2] = v0.z; L[3] = v0.w;
        L[4] = v1.x; L[5] = v1.y; L[6] = v1.z; L[7] = v1.w;
      }
      const int e0 = lane_in * 8;
      uint64_t key[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int e = e0 + q;
        key[q] = e < E ? ((uint64_t)ordered_key(L[q]) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)e)
                       : 0ull;
      }
      sort8_desc(key);
      float vals[kMaxTopK];
      int ids[kMaxTopK];
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) {
        vals[j] = 0.f;
        ids[j] = 0;
        if (j < k) {
          uint64_t best = key[0];
#pragma unroll
          for (int o = 1; o < G; o <<= 1) {
            const uint64_t other = __shfl_xor_sync(gmask, best, o);
            best = other > best ? other : best;
          }
          const bool pop = key[0] == best;   // keys are distinct but for absent experts
#pragma unroll
          for (int q = 0; q < 7; ++q) key[q] = pop ? key[q + 1] : key[q];
          key[7] = pop ? 0ull : key[7];
          const uint32_t kb = (uint32_t)(best >> 32);
          vals[j] = __uint_as_float((kb & 0x80000000u) ? (kb & 0x7FFFFFFFu) : ~kb);
          ids[j] = (int)(0xFFFFFFFFu - (uint32_t)(best & 0xFFFFFFFFull));
        }
      }
      const float m = vals[0];
      float p[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) p[q] = (e0 + q < E) ? expf(L[q] - m) : 0.f;
      float sum = ((p[0] + p[1]) + (p[2] + p[3])) + ((p[4] + p[5]) + (p[6] + p[7]));
#pragma unroll
      for (int o = 1; o < G; o <<= 1) sum += __shfl_xor_sync(gmask, sum, o);
      const float inv = __frcp_rn(sum);
      *reinterpret_cast<float4*>(row) = make_float4(p[0] * inv, p[1] * inv, p[2] * inv, p[3] * inv);
      *reinterpret_cast<float4*>(row + 4) =
          make_float4(p[4] * inv, p[5] * inv, p[6] * inv, p[7] * inv);
      if (lane_in == 0) {
        float ex[kMaxTopK];
        float sk = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
          ex[j] = j < k ? expf(vals[j] - vals[0]) : 0.f;
          sk += ex[j];
        }
        const float skinv = __frcp_rn(sk);
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j)
          if (j < k) {
            a.idx[(size_t)t * k + j] = ids[j];
            a.gates[(size_t)t * k + j] = ex[j] * skinv;
          }
      }
    }
  }
  __syncthreads();
  // Column sums of the probabilities over this CTA's tokens, in token order.
  if ((int)threadIdx.x < EP) {
    const int nvalid = min(rpc, T - (t_base + r0));
    float v = 0.f;
    for (int i = 0; i < nvalid; ++i) v += lg[(r0 + i) * S::LGS + threadIdx.x];
    csum[threadIdx.x] = v;
  }
  cluster.sync();
  if (rank == 0) {
    if ((int)threadIdx.x < E) {
      float v = 0.f;
      for (int sp = 0; sp < nsplit; ++sp) v += cluster.map_shared_rank(csum, sp)[threadIdx.x];
      a.part[(size_t)tile * E + threadIdx.x] = v;
      __threadfence();
    }
    // The last tile to finish turns the rows into P_e = (sum over rows in
    // fp64) / T: 256 fixed groups (group g of expert e adds rows g, g +
    // groups, ... in order; then the groups in order), whichever CTA is last.
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
      const unsigned ntiles = gridDim.x / (unsigned)nsplit;
      s_last = atomicAdd(a.done, 1u) == ntiles - 1u;
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      double* red = reinterpret_cast<double*>(lg);   // no CTA reads lg any more
      const int nrows = (int)(gridDim.x / (unsigned)nsplit);
      const int groups = max(1, 256 / E);
      for (int v = threadIdx.x; v < 256; v += TTHREADS) {
        const int e = v % E, g = v / E;
        double acc = 0.0;
        if (g < groups)
          for (int b = g; b < nrows; b += groups) acc += (double)__ldcg(a.part + (size_t)b * E + e);
        red[v] = acc;
      }
      __syncthreads();
      for (int e = threadIdx.x; e < E; e += TTHREADS) {
        double sum = 0.0;
        for (int gg = 0; gg < groups; ++gg)
          if (gg * E + e < 256) sum += red[gg * E + e];
        a.prob_mean[e] = T > 0 ? (float)(sum / (double)T) : 0.f;
      }
      if (threadIdx.x == 0) *a.done = 0u;            // ready for the next launch
    }
  }
teardown:
  cluster.sync();  // peers keep their shared memory until every read of it is done

  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, S::TMEM_COLS);
  }
}

// CTAs per token tile: doubled while the grid stays within one wave at two
// CTAs per SM and every CTA keeps at least four 64-wide d blocks (fewer
// leave each CTA's fixed start-up and finishing costs exposed), at most 8.
// Measured on B200 at T x d = 8192 x 4096, 16384 x 2048, 4096 x 768, 64 x
// 4096, 1024 x 4096 and 32768 x 4096: this picks the fastest of 1, 2, 4, 8.
int tc_splits(int tiles, int chunks) {
  const int slots = 2 * device_sm_count();
  int s = 1;
  while (s < 8 && tiles * 2 * s <= slots && chunks >= 4 * 2 * s) s *= 2;
  return s;
}

bool encode_bf16(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box) {
  const cuuint32_t estr[3] = {1, 1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank,
                              const_cast<void*>(ptr), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// W2: kModeNoisy's second weight matrix (W_noise), split into planes 3-5.
template <int EP, int MODE>
cudaError_t run_router_tc(const moe_config_t& c, const __nv_bfloat16* x, const float* W,
                          const float* W2, const TcArgs& a, __nv_bfloat16* w_split,
                          cudaStream_t s, int* tiles_out) {
  using S = TcShape<EP, MODE>;
  const int chunks = ceil_div(c.d, TBK);
  // kModeNoisy: a third plane of blocks draws z for every (token, expert)
  const NoiseDraw nd{const_cast<double*>(a.noise_z), a.seed, a.offset, a.token_base, c.T};
  const int zblocks = S::NOISY ? (int)std::min<long long>(((long long)c.T * c.E + 255) / 256,
                                                          (long long)device_sm_count() * 4)
                               : 0;
  cudaError_t e = launch_kernel(split_router_weights_kernel,
                                dim3(std::max(chunks, zblocks), S::TERMS / 3 + (S::NOISY ? 1 : 0)),
                                256, 0, s, 0, W, W2, c.d, c.E, EP, w_split, nd);
  if (e != cudaSuccess) return e;
  CUtensorMap tx, tw;
  const cuuint64_t xd[2] = {(cuuint64_t)c.d, (cuuint64_t)c.T};
  const cuuint64_t xs[1] = {(cuuint64_t)c.d * 2};
  const cuuint32_t xb[2] = {TBK, TBM};
  const cuuint64_t wd[3] = {(cuuint64_t)c.d, (cuuint64_t)EP, (cuuint64_t)S::TERMS};
  const cuuint64_t wstr[2] = {(cuuint64_t)c.d * 2, (cuuint64_t)EP * (cuuint64_t)c.d * 2};
  const cuuint32_t wb[3] = {TBK, EP, (cuuint32_t)S::TERMS};
  if (!encode_bf16(&tx, x, 2, xd, xs, xb) || !encode_bf16(&tw, w_split, 3, wd, wstr, wb))
    return cudaErrorInvalidValue;
  const int tiles = ceil_div(c.T, TBM);
  // the same split for every mode, so that the noisy router sums the logits
  // in the same order as the plain one
  const int nsplit = tc_splits(tiles, chunks);
  *tiles_out = tiles;
  auto kern = router_tc_kernel<EP, MODE>;
  e = ensure_smem_limit(reinterpret_cast<const void*>(kern), S::SMEM);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, tiles * nsplit, TTHREADS, S::SMEM, s, nsplit, tx, tw, a);
}

}  // namespace

cudaError_t launch_route_tc(const moe_config_t& c, const __nv_bfloat16* x, const float* W_router,
                            const float* bias, const float* noise, int32_t* idx, float* gates,
                            float* logits_out, float* router_part, __nv_bfloat16* w_split,
                            int32_t* err, cudaStream_t s, int* tiles_out, float* prob_mean,
                            unsigned* done) {
  if (tensor_map_encoder() == nullptr) return cudaErrorNotSupported;
  const TcArgs a{bias, noise, idx, gates, logits_out, router_part, err, c.T, c.d, c.E, c.top_k,
                 0, 0, 0, nullptr, nullptr, prob_mean, done};
  switch (router_tc_width(c)) {
    case 16: return run_router_tc<16, kModeRoute>(c, x, W_router, W_router, a, w_split, s, tiles_out);
    case 32: return run_router_tc<32, kModeRoute>(c, x, W_router, W_router, a, w_split, s, tiles_out);
    case 64: return run_router_tc<64, kModeRoute>(c, x, W_router, W_router, a, w_split, s, tiles_out);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_route_tc_noisy(const moe_config_t& c, const __nv_bfloat16* x,
                                  const float* W_router, const float* bias, const float* W_noise,
                                  uint64_t seed, uint64_t offset, long long token_base,
                                  int32_t* idx, float* gates, float* logits_out, float* noise_out,
                                  float* router_part, __nv_bfloat16* w_split, double* noise_z,
                                  int32_t* err, cudaStream_t s, int* tiles_out, float* prob_mean,
                                  unsigned* done) {
  if (tensor_map_encoder() == nullptr) return cudaErrorNotSupported;
  const TcArgs a{bias, nullptr, idx, gates, logits_out, router_part, err, c.T, c.d, c.E, c.top_k,
                 seed, offset, token_base, noise_out, noise_z, prob_mean, done};
  switch (router_tc_width(c)) {
    case 16: return run_router_tc<16, kModeNoisy>(c, x, W_router, W_noise, a, w_split, s, tiles_out);
    case 32: return run_router_tc<32, kModeNoisy>(c, x, W_router, W_noise, a, w_split, s, tiles_out);
    case 64: return run_router_tc<64, kModeNoisy>(c, x, W_router, W_noise, a, w_split, s, tiles_out);
    default: return cudaErrorInvalidValue;
  }
}

namespace {

// In place: noise logits l (T, E) -> z(token_base + t, e) * softplus(l)
// (gate_noise_value), one thread per element.
__global__ void __launch_bounds__(256)
    gate_noise_kernel(float* __restrict__ buf, long long n, int E, uint64_t seed, uint64_t offset,
                      long long token_base) {
  pdl_wait_and_release();
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long t = i / E;
    const int e = (int)(i - t * E);
    buf[i] = gate_noise_value(seed, offset, t + token_base, e, buf[i]);
  }
}

}  // namespace

cudaError_t launch_gate_noise(const moe_config_t& c, const __nv_bfloat16* x, const float* W_noise,
                              uint64_t seed, uint64_t offset, long long token_base,
                              float* noise_out, __nv_bfloat16* w_split, int32_t* err,
                              cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  if (tensor_map_encoder() == nullptr) return cudaErrorNotSupported;
  const TcArgs a{nullptr, nullptr, nullptr, nullptr, noise_out, nullptr, err, c.T, c.d, c.E,
                 c.top_k, 0, 0, 0, nullptr, nullptr, nullptr, nullptr};
  int tiles = 0;
  cudaError_t e;
  switch (router_tc_width(c)) {
    case 16: e = run_router_tc<16, kModeLogits>(c, x, W_noise, W_noise, a, w_split, s, &tiles); break;
    case 32: e = run_router_tc<32, kModeLogits>(c, x, W_noise, W_noise, a, w_split, s, &tiles); break;
    case 64: e = run_router_tc<64, kModeLogits>(c, x, W_noise, W_noise, a, w_split, s, &tiles); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  const long long n = (long long)c.T * c.E;
  const int blocks = (int)std::min<long long>((n + 255) / 256, (long long)device_sm_count() * 8);
  return launch_kernel(gate_noise_kernel, blocks, 256, 0, s, 0, noise_out, n, c.E, seed, offset,
                       token_base);
}

}  // namespace moe
