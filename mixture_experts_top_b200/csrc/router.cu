// router.cu - fused MoE router: fp32 logits, softmax, top-k, renormalised
// gates and per-CTA column sums of the probabilities.
//
// "Mixture-of-Experts Routing - LLM Internals" (mlgrind.dev), Algorithm 1-2:
//   logits = x @ W_router; probs = softmax(logits); indices = the k largest
//   logits by descending value, a stable order (lower index first on ties);
//   gates = softmax over the chosen k logits.
// "Mixture of Experts: the Sparsely-Gated Layer" (paperfordummies.in), The
// code, `router`: an optional per-expert bias, then optional noise, are added
// to the logits before the softmax and the top-k.
//
// This fp32 SIMT kernel serves fp32 tokens, more than 64 experts and
// moe_route_noalloc; bf16 tokens with E <= 64 take the tensor-core router of
// router_tc.cu (launch_route below picks).
//
// Design (B200): a thread-block cluster of S CTAs (S = 1..8) owns a tile of
// 32 or 64 tokens; each CTA of the cluster takes 1/S of the contraction
// range d.  The contraction x (tile, d/S) @ W (d/S, E) runs on the fp32 pipes
// (fp32 tokens have no exact bf16 tensor-core form): x and W stream through
// shared memory in k chunks with a multi-stage cp.async pipeline; each lane
// owns TM tokens and TN experts, so W values are warp-wide broadcasts and x
// rows are read as conflict-free 16-byte vectors (rows padded by 16 bytes).
// k is consumed in pairs with packed fp32 FMAs (fma.rn.f32x2): unpacking a
// 32-bit word of bf16 x gives the pair {x_k, x_k+1}, and W is stored
// interleaved by k pairs so one broadcast load feeds two experts.
// Warps split experts (WN) and the chunk (KS); the KS partial sums are added
// in a fixed order in shared memory.  Splitting d over the cluster keeps the
// serial chain of chunk loads per CTA short, so the kernel is not bound by
// one CTA's load latency when there are few tokens.  The S partial logit
// tiles are then added in rank order through distributed shared memory, and
// the cluster's warps finish one token each: bias and noise, max-subtracted
// softmax, k rounds of a warp-wide max over 64-bit keys (order-preserving
// logit bits, then the complemented expert index so the lower index wins
// ties), the gates, and a running per-lane sum of the probabilities.  The
// column sums are added across warps and CTAs in a fixed order into one row
// per token tile; a second small kernel adds the rows in fp64.
#include <cooperative_groups.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace cg = cooperative_groups;

namespace moe {
namespace {

// 16 bytes of x -> VEC/2 pairs {x_k, x_k+1} (fp32).
template <typename XT>
struct XVec;
template <>
struct XVec<float> {
  static constexpr int kN = 4;  // elements per 16 bytes
  __device__ static void load(const float* p, float2 (&v)[2]) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = make_float2(q.x, q.y);
    v[1] = make_float2(q.z, q.w);
  }
};
template <>
struct XVec<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ static void load(const __nv_bfloat16* p, float2 (&v)[4]) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      v[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
  }
};

__device__ __forceinline__ void cp_async_16(void* dst, const void* src, bool valid) {
  const uint32_t n = valid ? 16u : 0u;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_4(void* dst, const void* src, bool valid) {
  const uint32_t n = valid ? 4u : 0u;
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <typename XT>
struct RouterArgs {
  const XT* x;
  const float* W;
  const float* bias;
  const float* noise;
  int32_t* idx;
  float* gates;
  float* logits_out;
  float* part;
  int T, d, E, k;
};

constexpr int kMaxK = 8;

// TM tokens per lane (a CTA owns BM = 32 * TM tokens), TN experts per lane,
// WN warps across experts, KS warps across the k chunk, BK k per chunk,
// ST cp.async pipeline stages.
template <typename XT, int TM, int TN, int WN, int KS, int BK, int ST>
struct RouterShape {
  static constexpr int VEC = XVec<XT>::kN;
  static constexpr int BM = 32 * TM;
  static constexpr int EP = TN * WN;            // experts covered (padded E)
  static constexpr int THREADS = 32 * WN * KS;
  static constexpr int XROW = BK + VEC;         // padded x row, elements
  static constexpr int X_STAGE = BM * XROW;     // elements
  static constexpr int W_STAGE = BK * EP;       // floats
  static constexpr int PIPE_BYTES = ST * (X_STAGE * (int)sizeof(XT) + W_STAGE * 4);
  static constexpr int PART_BYTES = KS * BM * EP * 4;
  static constexpr int CS_BYTES = WN * KS * EP * 4;
  static constexpr int MAIN_BYTES = PIPE_BYTES > PART_BYTES ? PIPE_BYTES : PART_BYTES;
  static constexpr int SMEM = MAIN_BYTES + CS_BYTES;
  static_assert((BK / KS) % VEC == 0, "k split must hold whole vectors");
  static_assert(TN % 4 == 0, "experts per lane must be a multiple of 4");
  static_assert(BK % 2 == 0, "k is consumed in pairs");
  static_assert((EP & (EP - 1)) == 0, "the padded expert width is a power of two");
  static_assert(BM % kRouterTokens == 0, "CTA tiles are whole multiples of the sizing unit");
};

template <typename XT, int TM, int TN, int WN, int KS, int BK, int ST>
__global__ void __launch_bounds__(32 * WN * KS)
    router_kernel(const RouterArgs<XT> a) {
  pdl_wait_and_release();
  using S = RouterShape<XT, TM, TN, WN, KS, BK, ST>;
  constexpr int VEC = S::VEC, EP = S::EP, NT = S::THREADS, XROW = S::XROW, BM = S::BM;
  constexpr int QMAX = (EP + 31) / 32;  // experts per lane in the finishing pass
  extern __shared__ __align__(16) unsigned char smem[];
  XT* xs = reinterpret_cast<XT*>(smem);
  float* wsm = reinterpret_cast<float*>(smem + ST * S::X_STAGE * sizeof(XT));
  float* lg = reinterpret_cast<float*>(smem);                       // after the k loop
  float* cs = reinterpret_cast<float*>(smem + S::MAIN_BYTES);

  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int nsplit = (int)cluster.num_blocks();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wn = warp % WN, kg = warp / WN;
  const int T = a.T, d = a.d, E = a.E;
  const int tile = blockIdx.x / nsplit;
  const int t_base = tile * BM;
  // This CTA's share of the k chunks.
  const int total_chunks = (d + BK - 1) / BK;
  const int per = (total_chunks + nsplit - 1) / nsplit;
  const int c_begin = min(rank * per, total_chunks);
  const int nchunks = min(per, total_chunks - c_begin);

  // Padding columns e >= E of the W tiles are never loaded: zero them once.
  if (E < EP) {
    for (int i = tid; i < ST * S::W_STAGE; i += NT)
      if ((i >> 1) % EP >= E) wsm[i] = 0.f;
  }

  auto load_stage = [&](int chunk, int stage) {
    const int k0 = (c_begin + chunk) * BK;
    XT* xd = xs + stage * S::X_STAGE;
    constexpr int XV = BK / VEC;
    for (int v = tid; v < BM * XV; v += NT) {
      const int r = v / XV, cv = v % XV;
      const int t = t_base + r, kk = k0 + cv * VEC;
      const bool ok = (t < T) && (kk < d);
      cp_async_16(xd + r * XROW + cv * VEC, ok ? (const void*)(a.x + (size_t)t * d + kk) : (const void*)a.x, ok);
    }
    // W chunk rows k0..k0+BK-1, stored as [k/2][e][k%2] so that one 16-byte
    // broadcast load gives {W[k][e], W[k+1][e], W[k][e+1], W[k+1][e+1]}.
    // Indexed by the compile-time padded width EP (a power of two), so no
    // integer division by the runtime E; columns e >= E are skipped and keep
    // their zeros.
    float* wd = wsm + stage * S::W_STAGE;
#pragma unroll 4
    for (int v = tid; v < BK * EP; v += NT) {
      const int r = v / EP, c = v % EP, kk = k0 + r;
      if (c < E) {
        const bool ok = kk < d;
        cp_async_4(wd + ((r >> 1) * EP + c) * 2 + (r & 1),
                   ok ? (const void*)(a.W + (size_t)kk * E + c) : (const void*)a.W, ok);
      }
    }
  };

  // acc[m][n] holds the even-k and odd-k partial sums of token m, expert n.
  float2 acc[TM][TN];
#pragma unroll
  for (int m = 0; m < TM; ++m)
#pragma unroll
    for (int n = 0; n < TN; ++n) acc[m][n] = make_float2(0.f, 0.f);

  // Prologue: ST - 1 chunks in flight (one commit group per chunk; empty
  // groups past the end keep the group count uniform).
#pragma unroll
  for (int st = 0; st < ST - 1; ++st) {
    if (st < nchunks) load_stage(st, st);
    cp_async_commit();
  }
  for (int chunk = 0; chunk < nchunks; ++chunk) {
    cp_async_wait<ST - 2>();   // chunk `chunk` has landed
    __syncthreads();           // ... for every thread; stage (chunk-1)%ST is free
    const int nxt = chunk + ST - 1;
    if (nxt < nchunks) load_stage(nxt, nxt % ST);
    cp_async_commit();
    const int stage = chunk % ST;
    const XT* xa = xs + stage * S::X_STAGE + lane * XROW;
    const float* wb = wsm + stage * S::W_STAGE + wn * TN * 2;
#pragma unroll
    for (int kv = kg * (BK / KS); kv < (kg + 1) * (BK / KS); kv += VEC) {
      float2 xp[TM][VEC / 2];
#pragma unroll
      for (int m = 0; m < TM; ++m) XVec<XT>::load(xa + m * 32 * XROW + kv, xp[m]);
#pragma unroll
      for (int pi = 0; pi < VEC / 2; ++pi) {
        const float4* wr = reinterpret_cast<const float4*>(wb + ((kv >> 1) + pi) * EP * 2);
#pragma unroll
        for (int q = 0; q < TN / 2; ++q) {
          const float4 w = wr[q];
          const float2 w0 = make_float2(w.x, w.y), w1 = make_float2(w.z, w.w);
#pragma unroll
          for (int m = 0; m < TM; ++m) {
            acc[m][2 * q] = __ffma2_rn(xp[m][pi], w0, acc[m][2 * q]);
            acc[m][2 * q + 1] = __ffma2_rn(xp[m][pi], w1, acc[m][2 * q + 1]);
          }
        }
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // This CTA's partial logits: per k group to shared memory, then a
  // fixed-order sum over the groups into lg[BM][EP].
#pragma unroll
  for (int m = 0; m < TM; ++m) {
    float* p = lg + (kg * BM + m * 32 + lane) * EP + wn * TN;
#pragma unroll
    for (int n = 0; n < TN; ++n) p[n] = acc[m][n].x + acc[m][n].y;
  }
  __syncthreads();
  if (KS > 1) {
    for (int i = tid; i < BM * EP; i += NT) {
      float v = lg[i];
#pragma unroll
      for (int g = 1; g < KS; ++g) v += lg[g * BM * EP + i];
      lg[i] = v;
    }
  }
  cluster.sync();  // every CTA's partial tile is complete and visible

  // Finishing pass: token r of the tile is finished by CTA r % nsplit, one
  // warp per token; the logits are the rank-ordered sum of the partials.
  constexpr int NW = WN * KS;
  float colsum[QMAX];
#pragma unroll
  for (int q = 0; q < QMAX; ++q) colsum[q] = 0.f;
  const int k = a.k;
  for (int r = rank + nsplit * warp; r < BM; r += nsplit * NW) {
    const int t = t_base + r;
    if (t >= T) break;
    float L[QMAX];
    float m = -INFINITY;
#pragma unroll
    for (int q = 0; q < QMAX; ++q) {
      const int e = lane + 32 * q;
      float v = -INFINITY;
      if (e < E) {
        v = 0.f;
        for (int sp = 0; sp < nsplit; ++sp) v += cluster.map_shared_rank(lg, sp)[r * EP + e];
        if (a.bias != nullptr) v = __fadd_rn(v, a.bias[e]);
        if (a.noise != nullptr) v = __fadd_rn(v, a.noise[(size_t)t * E + e]);
        if (a.logits_out != nullptr) a.logits_out[(size_t)t * E + e] = v;
      }
      L[q] = v;
      m = fmaxf(m, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float p[QMAX];
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < QMAX; ++q) {
      p[q] = (lane + 32 * q < E) ? expf(L[q] - m) : 0.f;
      sum += p[q];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
#pragma unroll
    for (int q = 0; q < QMAX; ++q) colsum[q] += p[q] / sum;

    // Top-k over packed keys: (order-preserving logit bits) << 32 | ~e.
    uint64_t key[QMAX];
#pragma unroll
    for (int q = 0; q < QMAX; ++q) {
      const int e = lane + 32 * q;
      key[q] = (e < E) ? ((uint64_t)ordered_key(L[q]) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)e)
                       : 0ull;
    }
    float vals[kMaxK];
    int ids[kMaxK];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      vals[j] = 0.f;
      ids[j] = 0;
      if (j < k) {
        uint64_t best = 0ull;
#pragma unroll
        for (int q = 0; q < QMAX; ++q) best = key[q] > best ? key[q] : best;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
          best = other > best ? other : best;
        }
        ids[j] = (int)(0xFFFFFFFFu - (uint32_t)(best & 0xFFFFFFFFull));
        const uint32_t kb = (uint32_t)(best >> 32);
        vals[j] = __uint_as_float((kb & 0x80000000u) ? (kb & 0x7FFFFFFFu) : ~kb);
#pragma unroll
        for (int q = 0; q < QMAX; ++q)
          if (key[q] == best) key[q] = 0ull;
      }
    }
    float ex[kMaxK];
    float sk = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      ex[j] = (j < k) ? expf(vals[j] - vals[0]) : 0.f;
      sk += ex[j];
    }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j < k && lane == j) {
        a.idx[(size_t)t * k + j] = ids[j];
        a.gates[(size_t)t * k + j] = ex[j] / sk;
      }
    }
  }

  // Column sums of probs: per warp -> own shared memory; then CTA 0 adds
  // them over ranks and warps in a fixed order into this tile's row.
#pragma unroll
  for (int q = 0; q < QMAX; ++q) {
    const int e = lane + 32 * q;
    if (e < EP) cs[warp * EP + e] = colsum[q];
  }
  cluster.sync();
  if (rank == 0) {
    for (int e = tid; e < E; e += NT) {
      float v = 0.f;
      for (int sp = 0; sp < nsplit; ++sp) {
        const float* pcs = cluster.map_shared_rank(cs, sp);
        for (int w = 0; w < NW; ++w) v += pcs[w * EP + e];
      }
      a.part[(size_t)tile * E + e] = v;
    }
  }
  cluster.sync();  // peers keep their shared memory until CTA 0 has read it
}

// P_e = (sum over token tiles of the column-sum rows, in fp64) / T.  Each
// thread adds a fixed strided subset of rows in increasing order, then the
// subsets are added in increasing order.
__global__ void __launch_bounds__(256)
    prob_mean_kernel(const float* __restrict__ part, int nrows, int E, int T,
                     float* __restrict__ prob_mean) {
  pdl_wait_and_release();
  __shared__ double acc[256];
  const int groups = max(1, (int)blockDim.x / E);   // threads per expert
  const int e = threadIdx.x % E, g = threadIdx.x / E;
  double v = 0.0;
  if (g < groups)
    for (int b = g; b < nrows; b += groups) v += (double)part[(size_t)b * E + e];
  acc[threadIdx.x] = v;
  __syncthreads();
  for (int ee = threadIdx.x; ee < E; ee += blockDim.x) {
    double s = 0.0;
    for (int gg = 0; gg < groups; ++gg)
      if (gg * E + ee < (int)blockDim.x) s += acc[gg * E + ee];
    prob_mean[ee] = T > 0 ? (float)(s / (double)T) : 0.f;
  }
}

// Clusters of nsplit CTAs per token tile: enough CTAs to fill the GPU about
// four times over, at most 8 per cluster and at most one k chunk each.
int router_splits(int tiles, int chunks) {
  const int target = 4 * device_sm_count();
  int s = 1;
  while (s < 8 && tiles * s < target && s * 2 <= chunks) s *= 2;
  return s;
}

template <typename XT, int TM, int TN, int WN, int KS, int BK, int ST>
cudaError_t run_router(const RouterArgs<XT>& a, cudaStream_t s, int* tiles_out) {
  using S = RouterShape<XT, TM, TN, WN, KS, BK, ST>;
  auto kern = router_kernel<XT, TM, TN, WN, KS, BK, ST>;
  const int tiles = ceil_div(a.T, S::BM);
  const int nsplit = router_splits(tiles, ceil_div(a.d, BK));
  *tiles_out = tiles;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), S::SMEM);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, tiles * nsplit, S::THREADS, S::SMEM, s, nsplit, a);
}

// Two tokens per lane everywhere (each W broadcast feeds two packed FMAs);
// small E keeps 3 chunks in flight to stream x, large E narrows the chunk to
// bound shared memory.
template <typename XT>
cudaError_t dispatch_router(const RouterArgs<XT>& a, cudaStream_t s, int* tiles) {
  if (a.E <= 8) return run_router<XT, 2, 8, 1, 4, 64, 4>(a, s, tiles);
  if (a.E <= 16) return run_router<XT, 2, 8, 2, 2, 64, 4>(a, s, tiles);
  if (a.E <= 32) return run_router<XT, 2, 8, 4, 2, 64, 3>(a, s, tiles);
  if (a.E <= 64) return run_router<XT, 2, 8, 8, 1, 64, 2>(a, s, tiles);
  if (a.E <= 128) return run_router<XT, 2, 8, 16, 1, 32, 2>(a, s, tiles);
  return run_router<XT, 1, 16, 16, 1, 32, 2>(a, s, tiles);  // 512 threads: 128 regs each
}

}  // namespace

cudaError_t launch_prob_mean(const float* router_part, int rows, int E, int T, float* prob_mean,
                             cudaStream_t s) {
  return launch_kernel(prob_mean_kernel, 1, 256, 0, s, 0, router_part, rows, E, T, prob_mean);
}

cudaError_t launch_route(const moe_config_t& c, const void* x, const float* W_router,
                         const float* bias, const float* noise, int32_t* idx, float* gates,
                         float* prob_mean, float* logits_out, float* router_part,
                         __nv_bfloat16* w_split, int32_t* err, cudaStream_t s, unsigned* done) {
  int tiles = 0;  // token tiles; each writes one row of router_part
  if (c.T > 0) {
    cudaError_t e;
    if (w_split != nullptr && done != nullptr && router_tc_width(c) > 0) {
      // the tensor-core router writes P itself (its last tile)
      return launch_route_tc(c, static_cast<const __nv_bfloat16*>(x), W_router, bias, noise, idx,
                             gates, logits_out, router_part, w_split, err, s, &tiles, prob_mean,
                             done);
    } else if (c.act_dtype == MOE_BF16) {
      RouterArgs<__nv_bfloat16> a{static_cast<const __nv_bfloat16*>(x), W_router, bias, noise, idx,
                                  gates, logits_out, router_part, c.T, c.d, c.E, c.top_k};
      e = dispatch_router(a, s, &tiles);
    } else {
      RouterArgs<float> a{static_cast<const float*>(x), W_router, bias, noise, idx,
                          gates, logits_out, router_part, c.T, c.d, c.E, c.top_k};
      e = dispatch_router(a, s, &tiles);
    }
    if (e != cudaSuccess) return e;
  }
  return launch_kernel(prob_mean_kernel, 1, 256, 0, s, 0, router_part, tiles, c.E, c.T,
                       prob_mean);
}

}  // namespace moe
