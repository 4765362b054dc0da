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
// Design (B200): a CTA owns 64 tokens.  The contraction x (64, d) @ W (d, E)
// runs on the fp32 pipes (fp32 results are required, so no tensor cores):
// x and W stream through shared memory in 64-wide k chunks with cp.async
// double buffering; each lane owns two tokens and TN experts, so W values
// are warp-wide broadcasts and x rows are read as conflict-free 16-byte
// vectors (rows padded by 16 bytes).  Warps split experts (WN) and the k
// range (KS); the KS partial sums are added in a fixed order in shared
// memory.  Then one warp per token finishes the row in registers: bias and
// noise, max-subtracted softmax, k rounds of a warp-wide max over 64-bit
// keys (order-preserving logit bits, then the complemented expert index so
// the lower index wins ties), the gates, and a running per-lane sum of the
// probabilities.  Column sums are combined across warps in a fixed order and
// written per CTA; a second tiny kernel adds the CTA partials in fp64.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

template <typename XT>
struct XVec;
template <>
struct XVec<float> {
  static constexpr int kN = 4;  // elements per 16 bytes
  __device__ static void load(const float* p, float (&v)[4]) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  }
};
template <>
struct XVec<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 q = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
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

constexpr int kBM = kRouterTokens;   // tokens per CTA (two per lane)
constexpr int kStages = 2;
constexpr int kMaxK = 8;

template <typename XT, int TN, int WN, int KS, int BK>
struct RouterShape {
  static constexpr int VEC = XVec<XT>::kN;
  static constexpr int EP = TN * WN;            // experts covered (padded E)
  static constexpr int THREADS = 32 * WN * KS;
  static constexpr int XROW = BK + VEC;         // padded x row, elements
  static constexpr int X_STAGE = kBM * XROW;    // elements
  static constexpr int W_STAGE = BK * EP;       // floats
  static constexpr int PIPE_BYTES = kStages * (X_STAGE * (int)sizeof(XT) + W_STAGE * 4);
  static constexpr int PART_BYTES = KS * kBM * EP * 4;
  static constexpr int CS_BYTES = WN * KS * EP * 4;
  static constexpr int MAIN_BYTES = PIPE_BYTES > PART_BYTES ? PIPE_BYTES : PART_BYTES;
  static constexpr int SMEM = MAIN_BYTES + CS_BYTES;
  static_assert((BK / KS) % VEC == 0, "k split must hold whole vectors");
  static_assert(TN % 4 == 0, "experts per lane must be a multiple of 4");
};

template <typename XT, int TN, int WN, int KS, int BK>
__global__ void __launch_bounds__(32 * WN * KS)
    router_kernel(const RouterArgs<XT> a) {
  using S = RouterShape<XT, TN, WN, KS, BK>;
  constexpr int VEC = S::VEC, EP = S::EP, NT = S::THREADS, XROW = S::XROW;
  constexpr int QMAX = (EP + 31) / 32;  // experts per lane in the finishing pass
  extern __shared__ __align__(16) unsigned char smem[];
  XT* xs = reinterpret_cast<XT*>(smem);
  float* wsm = reinterpret_cast<float*>(smem + kStages * S::X_STAGE * sizeof(XT));
  float* lg = reinterpret_cast<float*>(smem);                       // after the k loop
  float* cs = reinterpret_cast<float*>(smem + S::MAIN_BYTES);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wn = warp % WN, kg = warp / WN;
  const int T = a.T, d = a.d, E = a.E;
  const int t_base = blockIdx.x * kBM;
  const int nchunks = (d + BK - 1) / BK;

  // Padding columns e >= E of the W tiles are never loaded: zero them once.
  if (E < EP) {
    for (int i = tid; i < kStages * S::W_STAGE; i += NT)
      if (i % EP >= E) wsm[i] = 0.f;
  }

  auto load_stage = [&](int chunk, int stage) {
    const int k0 = chunk * BK;
    XT* xd = xs + stage * S::X_STAGE;
    constexpr int XV = BK / VEC;
    for (int v = tid; v < kBM * XV; v += NT) {
      const int r = v / XV, cv = v % XV;
      const int t = t_base + r, kk = k0 + cv * VEC;
      const bool ok = (t < T) && (kk < d);
      cp_async_16(xd + r * XROW + cv * VEC, ok ? (const void*)(a.x + (size_t)t * d + kk) : (const void*)a.x, ok);
    }
    float* wd = wsm + stage * S::W_STAGE;
    if ((E & 3) == 0) {
      const int EV = E >> 2;
      for (int v = tid; v < BK * EV; v += NT) {
        const int r = v / EV, cv = v % EV, kk = k0 + r;
        const bool ok = kk < d;
        cp_async_16(wd + r * EP + cv * 4, ok ? (const void*)(a.W + (size_t)kk * E + cv * 4) : (const void*)a.W, ok);
      }
    } else {
      for (int v = tid; v < BK * E; v += NT) {
        const int r = v / E, c = v % E, kk = k0 + r;
        const bool ok = kk < d;
        cp_async_4(wd + r * EP + c, ok ? (const void*)(a.W + (size_t)kk * E + c) : (const void*)a.W, ok);
      }
    }
    cp_async_commit();
  };

  float acc0[TN], acc1[TN];
#pragma unroll
  for (int n = 0; n < TN; ++n) acc0[n] = acc1[n] = 0.f;

  if (nchunks > 0) load_stage(0, 0);
  for (int chunk = 0; chunk < nchunks; ++chunk) {
    if (chunk + 1 < nchunks) {
      load_stage(chunk + 1, (chunk + 1) % kStages);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int stage = chunk % kStages;
    const XT* xa = xs + stage * S::X_STAGE + lane * XROW;
    const XT* xb = xa + 32 * XROW;
    const float* wb = wsm + stage * S::W_STAGE + wn * TN;
#pragma unroll
    for (int kv = kg * (BK / KS); kv < (kg + 1) * (BK / KS); kv += VEC) {
      float x0[VEC], x1[VEC];
      XVec<XT>::load(xa + kv, x0);
      XVec<XT>::load(xb + kv, x1);
#pragma unroll
      for (int u = 0; u < VEC; ++u) {
        const float4* wr = reinterpret_cast<const float4*>(wb + (kv + u) * EP);
#pragma unroll
        for (int q = 0; q < TN / 4; ++q) {
          const float4 w = wr[q];
          acc0[4 * q + 0] = fmaf(x0[u], w.x, acc0[4 * q + 0]);
          acc0[4 * q + 1] = fmaf(x0[u], w.y, acc0[4 * q + 1]);
          acc0[4 * q + 2] = fmaf(x0[u], w.z, acc0[4 * q + 2]);
          acc0[4 * q + 3] = fmaf(x0[u], w.w, acc0[4 * q + 3]);
          acc1[4 * q + 0] = fmaf(x1[u], w.x, acc1[4 * q + 0]);
          acc1[4 * q + 1] = fmaf(x1[u], w.y, acc1[4 * q + 1]);
          acc1[4 * q + 2] = fmaf(x1[u], w.z, acc1[4 * q + 2]);
          acc1[4 * q + 3] = fmaf(x1[u], w.w, acc1[4 * q + 3]);
        }
      }
    }
    __syncthreads();
  }

  // Partial logits of each k group -> shared memory, then a fixed-order sum.
  {
    float* p0 = lg + (kg * kBM + lane) * EP + wn * TN;
    float* p1 = p0 + 32 * EP;
#pragma unroll
    for (int n = 0; n < TN; ++n) {
      p0[n] = acc0[n];
      p1[n] = acc1[n];
    }
  }
  __syncthreads();
  if (KS > 1) {
    for (int i = tid; i < kBM * EP; i += NT) {
      float s = lg[i];
#pragma unroll
      for (int g = 1; g < KS; ++g) s += lg[g * kBM * EP + i];
      lg[i] = s;
    }
    __syncthreads();
  }

  // One warp per token: bias, noise, softmax, top-k, gates, column sums.
  constexpr int NW = WN * KS;
  float colsum[QMAX];
#pragma unroll
  for (int q = 0; q < QMAX; ++q) colsum[q] = 0.f;
  const int k = a.k;
  for (int r = warp; r < kBM; r += NW) {
    const int t = t_base + r;
    if (t >= T) break;
    float L[QMAX];
    float m = -INFINITY;
#pragma unroll
    for (int q = 0; q < QMAX; ++q) {
      const int e = lane + 32 * q;
      float v = -INFINITY;
      if (e < E) {
        v = lg[r * EP + e];
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
    float s = 0.f;
#pragma unroll
    for (int q = 0; q < QMAX; ++q) {
      p[q] = (lane + 32 * q < E) ? expf(L[q] - m) : 0.f;
      s += p[q];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
#pragma unroll
    for (int q = 0; q < QMAX; ++q) colsum[q] += p[q] / s;

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

  // Column sums of probs: per warp -> shared -> fixed-order sum over warps.
#pragma unroll
  for (int q = 0; q < QMAX; ++q) {
    const int e = lane + 32 * q;
    if (e < EP) cs[warp * EP + e] = colsum[q];
  }
  __syncthreads();
  for (int e = tid; e < E; e += NT) {
    float s = 0.f;
    for (int w = 0; w < NW; ++w) s += cs[w * EP + e];
    a.part[(size_t)blockIdx.x * E + e] = s;
  }
}

// P_e = (sum over router CTAs of the partial column sums, in fp64) / T.
__global__ void prob_mean_kernel(const float* __restrict__ part, int nblocks, int E, int T,
                                 float* __restrict__ prob_mean) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    double s = 0.0;
    for (int b = 0; b < nblocks; ++b) s += (double)part[(size_t)b * E + e];
    prob_mean[e] = T > 0 ? (float)(s / (double)T) : 0.f;
  }
}

template <typename XT, int TN, int WN, int KS, int BK>
cudaError_t run_router(const RouterArgs<XT>& a, int nblocks, cudaStream_t s) {
  using S = RouterShape<XT, TN, WN, KS, BK>;
  auto kern = router_kernel<XT, TN, WN, KS, BK>;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<nblocks, S::THREADS, S::SMEM, s>>>(a);
  return cudaGetLastError();
}

template <typename XT>
cudaError_t dispatch_router(const RouterArgs<XT>& a, int nblocks, cudaStream_t s) {
  if (a.E <= 8) return run_router<XT, 8, 1, 4, 64>(a, nblocks, s);
  if (a.E <= 16) return run_router<XT, 16, 1, 4, 64>(a, nblocks, s);
  if (a.E <= 32) return run_router<XT, 16, 2, 2, 64>(a, nblocks, s);
  if (a.E <= 64) return run_router<XT, 16, 4, 2, 64>(a, nblocks, s);
  if (a.E <= 128) return run_router<XT, 16, 8, 1, 32>(a, nblocks, s);
  return run_router<XT, 16, 16, 1, 32>(a, nblocks, s);
}

}  // namespace

cudaError_t launch_route(const moe_config_t& c, const void* x, const float* W_router,
                         const float* bias, const float* noise, int32_t* idx, float* gates,
                         float* prob_mean, float* logits_out, float* router_part,
                         cudaStream_t s) {
  const int nblocks = ceil_div(c.T, kRouterTokens);
  if (nblocks > 0) {
    cudaError_t e;
    if (c.act_dtype == MOE_BF16) {
      RouterArgs<__nv_bfloat16> a{static_cast<const __nv_bfloat16*>(x), W_router, bias, noise, idx,
                                  gates, logits_out, router_part, c.T, c.d, c.E, c.top_k};
      e = dispatch_router(a, nblocks, s);
    } else {
      RouterArgs<float> a{static_cast<const float*>(x), W_router, bias, noise, idx,
                          gates, logits_out, router_part, c.T, c.d, c.E, c.top_k};
      e = dispatch_router(a, nblocks, s);
    }
    if (e != cudaSuccess) return e;
  }
  prob_mean_kernel<<<1, 256, 0, s>>>(router_part, nblocks, c.E, c.T, prob_mean);
  return cudaGetLastError();
}

}  // namespace moe
