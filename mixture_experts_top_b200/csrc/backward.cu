// backward.cu - gradients of the routing half of the layer: the combine and
// the router (gates, and the load-balancing loss through P).
//
// The forward is "Mixture-of-Experts Routing - LLM Internals" (mlgrind.dev),
// Algorithm 2-4: gates = softmax over the chosen k logits, y_t = sum_j
// gates[t,j] * expert_{idx[t,j]}(x_t), aux = E * sum_e f_e * P_e.  f counts
// routing slots and carries no gradient ("Mixture of Experts: the
// Sparsely-Gated Layer", paperfordummies.in, The code, `switch_balance_loss`);
// P_e is the batch mean of softmax(logits)[:, e] and does.
//
//   combine:  dY[dest[t,j]] = g_tj dy_t,   dg_tj = <dy_t, Y[dest[t,j]]>
//             (a dropped slot: no row, dg = 0)
//   gates:    dL_tm += g_tm (dg_tm - sum_j g_tj dg_tj)      (m chosen)
//   aux:      dL_te += p_te (a_e - sum_e' p_te' a_e'),  a_e = daux E f_e / T_batch
//   logits:   L = x W (+ bias + noise):  dx = dL W^T,  dW = x^T dL,  dbias = sum_t dL
//
// All in fp32 with fixed summation orders (no atomics): the combine and the
// logit gradient one warp per token; dx one thread per column and 16 tokens,
// the E terms in order; dW and dbias as per-chunk partial sums over token
// chunks (tokens in order), then the chunks added in order.  Everything here
// is bound by HBM or by launch latency.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 q = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// One warp per token; 8 columns per lane step.  dgates: per lane partial
// dot products in column order, then a fixed butterfly over the warp.
template <typename InT>
__global__ void __launch_bounds__(256)
    combine_backward_kernel(const InT* __restrict__ dy, const float* __restrict__ y_perm,
                            const int32_t* __restrict__ dest, const float* __restrict__ gates,
                            float* __restrict__ dy_perm, float* __restrict__ dgates, int T, int k,
                            int d_out) {
  pdl_wait_and_release();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int nvec = d_out / 8;
  for (int t = gw; t < T; t += nw) {
    int dl = -1;
    float gl = 0.f;
    if (lane < k) {
      dl = dest[(size_t)t * k + lane];
      gl = gates[(size_t)t * k + lane];
    }
    int dj[8];
    float gj[8], part[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      dj[j] = __shfl_sync(0xffffffffu, dl, j);
      gj[j] = __shfl_sync(0xffffffffu, gl, j);
      part[j] = 0.f;
    }
    const InT* dyr = dy + (size_t)t * d_out;
    for (int v = lane; v < nvec; v += 32) {
      float g8[8];
      load8(dyr + (size_t)v * 8, g8);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k && dj[j] >= 0) {
          float y8[8];
          load8(y_perm + (size_t)dj[j] * d_out + (size_t)v * 8, y8);
#pragma unroll
          for (int i = 0; i < 8; ++i) part[j] = fmaf(g8[i], y8[i], part[j]);
          float4* o = reinterpret_cast<float4*>(dy_perm + (size_t)dj[j] * d_out + (size_t)v * 8);
          o[0] = make_float4(gj[j] * g8[0], gj[j] * g8[1], gj[j] * g8[2], gj[j] * g8[3]);
          o[1] = make_float4(gj[j] * g8[4], gj[j] * g8[5], gj[j] * g8[6], gj[j] * g8[7]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part[j] += __shfl_xor_sync(0xffffffffu, part[j], o);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k && lane == j) dgates[(size_t)t * k + j] = dj[j] >= 0 ? part[j] : 0.f;
  }
}

constexpr int kQMax = 8;  // experts per lane (E <= 256)

// One warp per token: the logit gradient of the gates and of aux.
__global__ void __launch_bounds__(256)
    route_dlogits_kernel(const float* __restrict__ logits, const int32_t* __restrict__ idx,
                         const float* __restrict__ gates, const float* __restrict__ dgates,
                         const float* __restrict__ f, const float* __restrict__ daux, int T, int E,
                         int k, double aux_scale, float* __restrict__ dlogits) {
  pdl_wait_and_release();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  // a_e = daux * E * f_e / T_batch (aux_scale = E / T_batch)
  float a[kQMax];
  const double da = (double)daux[0];
#pragma unroll
  for (int q = 0; q < kQMax; ++q) {
    const int e = lane + 32 * q;
    a[q] = e < E ? (float)(da * aux_scale * (double)f[e]) : 0.f;
  }
  for (int t = gw; t < T; t += nw) {
    const float* Lr = logits + (size_t)t * E;
    float L[kQMax], p[kQMax];
    float m = -INFINITY;
#pragma unroll
    for (int q = 0; q < kQMax; ++q) {
      const int e = lane + 32 * q;
      L[q] = e < E ? Lr[e] : -INFINITY;
      m = fmaxf(m, L[q]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = 0.f;
#pragma unroll
    for (int q = 0; q < kQMax; ++q) {
      p[q] = lane + 32 * q < E ? expf(L[q] - m) : 0.f;
      sum += p[q];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    float pa = 0.f;
#pragma unroll
    for (int q = 0; q < kQMax; ++q) {
      p[q] = p[q] / sum;
      pa = fmaf(p[q], a[q], pa);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) pa += __shfl_xor_sync(0xffffffffu, pa, o);
    // gate part: s = sum_j g_j dg_j over the chosen k
    float gj = 0.f, dgj = 0.f;
    int ej = -1;
    if (lane < k) {
      gj = gates[(size_t)t * k + lane];
      dgj = dgates[(size_t)t * k + lane];
      ej = idx[(size_t)t * k + lane];
    }
    float s = gj * dgj;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float term = gj * (dgj - s);
    float dl[kQMax];
#pragma unroll
    for (int q = 0; q < kQMax; ++q) dl[q] = p[q] * (a[q] - pa);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = __shfl_sync(0xffffffffu, ej, j);
      const float tj = __shfl_sync(0xffffffffu, term, j);
      if (j < k && e >= 0 && e < E && (e & 31) == lane) {
#pragma unroll
        for (int q = 0; q < kQMax; ++q)
          if (e >> 5 == q) dl[q] += tj;
      }
    }
    float* out = dlogits + (size_t)t * E;
#pragma unroll
    for (int q = 0; q < kQMax; ++q)
      if (lane + 32 * q < E) out[lane + 32 * q] = dl[q];
  }
}

// dx[t, c] = sum_e dL[t, e] W[c, e], e in increasing order.  A CTA owns 256
// columns and kTg tokens; W and dL stream through shared memory 32 experts
// at a time, so each thread keeps kTg accumulators for its column.
constexpr int kTg = 16;
constexpr int kEb = 32;

__global__ void __launch_bounds__(256)
    route_dx_kernel(const float* __restrict__ dlogits, const float* __restrict__ W, int T, int d,
                    int E, float* __restrict__ dx) {
  pdl_wait_and_release();
  __shared__ float ws[kEb][256];
  __shared__ float dls[kTg][kEb];
  const int c = blockIdx.x * 256 + threadIdx.x;
  // Token groups are strided over grid.y (at most 65535 rows of CTAs), so
  // any T is covered; each group's arithmetic is unchanged.
  const int ngroups = (T + kTg - 1) / kTg;
  for (int tg = blockIdx.y; tg < ngroups; tg += gridDim.y) {
    const int t0 = tg * kTg;
    float acc[kTg];
#pragma unroll
    for (int i = 0; i < kTg; ++i) acc[i] = 0.f;
    for (int e0 = 0; e0 < E; e0 += kEb) {
      __syncthreads();
      for (int i = threadIdx.x; i < kEb * 256; i += 256) {
        const int e = i / 256, cc = blockIdx.x * 256 + i % 256;
        ws[e][i % 256] = (e0 + e < E && cc < d) ? W[(size_t)cc * E + e0 + e] : 0.f;
      }
      for (int i = threadIdx.x; i < kTg * kEb; i += 256) {
        const int tt = i / kEb, e = i % kEb;
        dls[tt][e] = (t0 + tt < T && e0 + e < E) ? dlogits[(size_t)(t0 + tt) * E + e0 + e] : 0.f;
      }
      __syncthreads();
      const int ne = min(kEb, E - e0);
      for (int e = 0; e < ne; ++e) {
        const float wv = ws[e][threadIdx.x];
#pragma unroll
        for (int i = 0; i < kTg; ++i) acc[i] = fmaf(dls[i][e], wv, acc[i]);
      }
    }
    if (c < d)
#pragma unroll
      for (int i = 0; i < kTg; ++i)
        if (t0 + i < T) dx[(size_t)(t0 + i) * d + c] = acc[i];
  }
}

constexpr int kCt = 64;           // columns of x per dW CTA
constexpr int kTs = 32;           // tokens staged in shared memory at a time

// Partial dW and dbias over one chunk of tokens.  CTA (tile, chunk) owns
// columns [64 tile, 64 tile + 64) of x: thread (c, g) accumulates
// dW[c, e] for the experts e of group g (EPT of them), over the chunk's
// tokens in increasing order, x and dL staged 32 tokens at a time.  Tile 0
// also sums dL over the chunk for dbias.
template <typename XT, int EPT>
__global__ void __launch_bounds__(256)
    route_dw_partial_kernel(const XT* __restrict__ x, const float* __restrict__ dlogits, int T,
                            int d, int E, int nchunks, float* __restrict__ dw_part,
                            float* __restrict__ dbias_part) {
  pdl_wait_and_release();
  __shared__ float xs[kTs][kCt];
  extern __shared__ float dls[];   // [kTs][E]
  const int chunk = blockIdx.y;
  const int t0 = (int)((long long)T * chunk / nchunks);
  const int t1 = (int)((long long)T * (chunk + 1) / nchunks);
  const int cl = threadIdx.x % kCt, grp = threadIdx.x / kCt;   // 4 groups of experts
  const int c = blockIdx.x * kCt + cl;
  const int ebase = grp * EPT;
  float acc[EPT];
#pragma unroll
  for (int i = 0; i < EPT; ++i) acc[i] = 0.f;
  float bacc = 0.f;
  const bool do_bias = blockIdx.x == 0 && (int)threadIdx.x < E;
  for (int ts0 = t0; ts0 < t1; ts0 += kTs) {
    const int n = min(kTs, t1 - ts0);
    __syncthreads();
    for (int i = threadIdx.x; i < kTs * kCt; i += 256) {
      const int tt = i / kCt, cc = blockIdx.x * kCt + i % kCt;
      xs[tt][i % kCt] = (tt < n && cc < d) ? static_cast<float>(x[(size_t)(ts0 + tt) * d + cc])
                                          : 0.f;
    }
    for (int i = threadIdx.x; i < kTs * E; i += 256) {
      const int tt = i / E;
      dls[i] = tt < n ? dlogits[(size_t)(ts0 + tt) * E + (i - tt * E)] : 0.f;
    }
    __syncthreads();
    for (int tt = 0; tt < n; ++tt) {
      const float xv = xs[tt][cl];
      const float* dl = dls + tt * E + ebase;
#pragma unroll
      for (int i = 0; i < EPT; ++i)
        if (ebase + i < E) acc[i] = fmaf(xv, dl[i], acc[i]);
      if (do_bias) bacc += dls[tt * E + threadIdx.x];
    }
  }
  const long long total = (long long)d * E;
  if (c < d)
#pragma unroll
    for (int i = 0; i < EPT; ++i)
      if (ebase + i < E) dw_part[(size_t)chunk * total + (size_t)c * E + ebase + i] = acc[i];
  if (do_bias) dbias_part[(size_t)chunk * E + threadIdx.x] = bacc;
}

// dx for E <= 16 and d a multiple of 4: a thread owns 4 consecutive columns
// and keeps their 4 rows of W (4 x E values) in registers; CTA row y walks
// a contiguous range of tokens, their logit gradients staged 256 tokens at
// a time in shared memory (read by the whole warp from one address), and
// writes each token's 4 columns as one 16-byte store, so a warp writes 512
// contiguous bytes per token.  The arithmetic is route_dx_kernel's: e in
// increasing order from 0.
template <int EMAX>
__global__ void __launch_bounds__(256)
    route_dx_narrow_kernel(const float* __restrict__ dlogits, const float* __restrict__ W, int T,
                           int d, int E, float* __restrict__ dx) {
  pdl_wait_and_release();
  __shared__ float dls[256 * EMAX];
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  const bool active = c < d;
  // this thread's 4 rows of W are 4 E contiguous floats
  float w[4][EMAX];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < EMAX; ++e) w[i][e] = 0.f;
  if (active) {
    const float* src = W + (size_t)c * E;
    if (E % 4 == 0 && (reinterpret_cast<uintptr_t>(W) & 15u) == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < EMAX / 4; ++q)
          if (4 * q < E) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(src + i * E) + q);
            w[i][4 * q] = v.x; w[i][4 * q + 1] = v.y; w[i][4 * q + 2] = v.z; w[i][4 * q + 3] = v.w;
          }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < EMAX; ++e)
          if (e < E) w[i][e] = __ldg(src + i * E + e);
    }
  }
  const int t0 = (int)((long long)T * blockIdx.y / gridDim.y);
  const int t1 = (int)((long long)T * (blockIdx.y + 1) / gridDim.y);
  for (int tb = t0; tb < t1; tb += 256) {
    const int n = min(256, t1 - tb);
    __syncthreads();
    // rows padded to EMAX, so a token's gradients are EMAX / 4 aligned vector loads
    for (int i = threadIdx.x; i < n * EMAX; i += blockDim.x) {
      const int tt = i / EMAX, e = i % EMAX;
      dls[i] = e < E ? dlogits[(size_t)(tb + tt) * E + e] : 0.f;
    }
    __syncthreads();
    if (!active) continue;
    for (int tt = 0; tt < n; ++tt) {
      float g[EMAX];
#pragma unroll
      for (int q = 0; q < EMAX / 4; ++q) {
        const float4 v = reinterpret_cast<const float4*>(dls + tt * EMAX)[q];
        g[4 * q] = v.x; g[4 * q + 1] = v.y; g[4 * q + 2] = v.z; g[4 * q + 3] = v.w;
      }
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < EMAX; ++e)
        if (e < E) {
          const float ge = g[e];
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[i] = fmaf(ge, w[i][e], acc[i]);
        }
      *reinterpret_cast<float4*>(dx + (size_t)(tb + tt) * d + c) =
          make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
  }
}

__device__ __forceinline__ void load_cols(const __nv_bfloat16* p, float* v, int n) {
  // n = 4 or 8 consecutive bf16 values (8 or 16 bytes)
  if (n == 8) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    const uint2 q = __ldg(reinterpret_cast<const uint2*>(p));
    v[0] = __uint_as_float(q.x << 16);
    v[1] = __uint_as_float(q.x & 0xFFFF0000u);
    v[2] = __uint_as_float(q.y << 16);
    v[3] = __uint_as_float(q.y & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load_cols(const float* p, float* v, int n) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  if (n == 8) {
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// Partial dW and dbias over one chunk of tokens for E <= 16 and d a
// multiple of CPT: a thread owns CPT consecutive columns of x and keeps
// CPT x E accumulators, reading x straight from global memory (a warp reads
// 32 * CPT contiguous elements of a row) with kDwAhead tokens' loads in
// flight; the chunk's logit gradients are staged 256 tokens at a time in
// shared memory.  The arithmetic is route_dw_partial_kernel's: tokens of the
// chunk in increasing order, each an fp32 FMA.
constexpr int kDwAhead = 2;
template <typename XT, int EMAX, int CPT>
__global__ void __launch_bounds__(256)
    route_dw_narrow_kernel(const XT* __restrict__ x, const float* __restrict__ dlogits, int T,
                           int d, int E, int nchunks, float* __restrict__ dw_part,
                           float* __restrict__ dbias_part) {
  pdl_wait_and_release();
  __shared__ float dls[256 * EMAX];
  const int chunk = blockIdx.y;
  const int t0 = (int)((long long)T * chunk / nchunks);
  const int t1 = (int)((long long)T * (chunk + 1) / nchunks);
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * CPT;
  const bool active = c < d;
  const bool do_bias = blockIdx.x == 0 && (int)threadIdx.x < E;
  float acc[CPT][EMAX];
#pragma unroll
  for (int i = 0; i < CPT; ++i)
#pragma unroll
    for (int e = 0; e < EMAX; ++e) acc[i][e] = 0.f;
  float bacc = 0.f;
  for (int tb = t0; tb < t1; tb += 256) {
    const int n = min(256, t1 - tb);
    __syncthreads();
    // rows padded to EMAX, so a token's gradients are EMAX / 4 aligned vector loads
    for (int i = threadIdx.x; i < n * EMAX; i += blockDim.x) {
      const int tt = i / EMAX, e = i % EMAX;
      dls[i] = e < E ? dlogits[(size_t)(tb + tt) * E + e] : 0.f;
    }
    __syncthreads();
    if (do_bias)
      for (int tt = 0; tt < n; ++tt) bacc += dls[tt * EMAX + threadIdx.x];
    if (!active) continue;
    // the next kDwAhead tokens' x is loaded while the current ones are used
    float xv[2][kDwAhead][CPT];
#pragma unroll
    for (int u = 0; u < kDwAhead; ++u)
      if (u < n) load_cols(x + (size_t)(tb + u) * d + c, xv[0][u], CPT);
    for (int tt0 = 0; tt0 < n; tt0 += 2 * kDwAhead) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int base = tt0 + half * kDwAhead;
        if (base >= n) break;
        const int nb = base + kDwAhead;
#pragma unroll
        for (int u = 0; u < kDwAhead; ++u)
          if (nb + u < n) load_cols(x + (size_t)(tb + nb + u) * d + c, xv[half ^ 1][u], CPT);
#pragma unroll
        for (int u = 0; u < kDwAhead; ++u)
          if (base + u < n) {
            float g[EMAX];
#pragma unroll
            for (int q = 0; q < EMAX / 4; ++q) {
              const float4 v = reinterpret_cast<const float4*>(dls + (base + u) * EMAX)[q];
              g[4 * q] = v.x; g[4 * q + 1] = v.y; g[4 * q + 2] = v.z; g[4 * q + 3] = v.w;
            }
#pragma unroll
            for (int e = 0; e < EMAX; ++e)
              if (e < E) {
#pragma unroll
                for (int i = 0; i < CPT; ++i) acc[i][e] = fmaf(xv[half][u][i], g[e], acc[i][e]);
              }
          }
      }
    }
  }
  const long long total = (long long)d * E;
  if (active)
#pragma unroll
    for (int i = 0; i < CPT; ++i)
#pragma unroll
      for (int e = 0; e < EMAX; ++e)
        if (e < E) dw_part[(size_t)chunk * total + (size_t)(c + i) * E + e] = acc[i][e];
  if (do_bias) dbias_part[(size_t)chunk * E + threadIdx.x] = bacc;
}

// Chunks added in increasing order.
__global__ void __launch_bounds__(256)
    route_dw_reduce_kernel(const float* __restrict__ dw_part, const float* __restrict__ dbias_part,
                           long long total, int E, int nchunks, float* __restrict__ dW,
                           float* __restrict__ dbias) {
  pdl_wait_and_release();
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    // 16 chunks' loads in flight at a time, added in chunk order
    float v = 0.f;
    for (int c0 = 0; c0 < nchunks; c0 += 16) {
      float t[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        t[u] = c0 + u < nchunks ? dw_part[(size_t)(c0 + u) * total + i] : 0.f;
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (c0 + u < nchunks) v += t[u];
    }
    dW[i] = v;
  }
  if (dbias != nullptr && blockIdx.x == 0)
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      float v = 0.f;
      for (int c = 0; c < nchunks; ++c) v += dbias_part[(size_t)c * E + e];
      dbias[e] = v;
    }
}

}  // namespace

// Token chunks of the dW partial sums: up to 128 of at least 64 tokens where
// E <= 16 (the narrow kernels: enough CTAs to stream x at HBM rate, and the
// partials stay small), else up to 16 of at least 128 tokens.
int route_backward_chunks(int T, int E) {
  return E <= 16 ? std::max(1, std::min(128, ceil_div(T, 64)))
                 : std::max(1, std::min(16, ceil_div(T, 128)));
}

cudaError_t launch_combine_backward(const moe_config_t& c, const void* dy, const float* y_perm,
                                    const int32_t* dest, const float* gates, float* dy_perm,
                                    float* dgates, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  const int blocks = std::min(ceil_div(c.T, 8), device_sm_count() * 16);
  if (c.act_dtype == MOE_BF16)
    return launch_kernel(combine_backward_kernel<__nv_bfloat16>, blocks, 256, 0, s, 0,
                         static_cast<const __nv_bfloat16*>(dy), y_perm, dest, gates, dy_perm,
                         dgates, c.T, c.top_k, c.d_out);
  return launch_kernel(combine_backward_kernel<float>, blocks, 256, 0, s, 0,
                       static_cast<const float*>(dy), y_perm, dest, gates, dy_perm, dgates, c.T,
                       c.top_k, c.d_out);
}

cudaError_t launch_route_backward(const moe_config_t& c, const void* x, const float* W,
                                  const float* logits, const int32_t* idx, const float* gates,
                                  const float* f, const float* dgates, const float* daux,
                                  int T_batch, float* dx, float* dW, float* dbias,
                                  float* dlogits, float* dw_part, float* dbias_part,
                                  cudaStream_t s) {
  const long long total = (long long)c.d * c.E;
  if (c.T == 0) {
    // no tokens: every gradient is zero
    cudaError_t e = cudaMemsetAsync(dW, 0, (size_t)total * 4, s);
    if (e == cudaSuccess && dbias != nullptr) e = cudaMemsetAsync(dbias, 0, (size_t)c.E * 4, s);
    return e;
  }
  const int wblocks = std::min(ceil_div(c.T, 8), device_sm_count() * 16);
  cudaError_t e = launch_kernel(route_dlogits_kernel, wblocks, 256, 0, s, 0, logits, idx, gates,
                                dgates, f, daux, c.T, c.E, c.top_k,
                                (double)c.E / (double)T_batch, dlogits);
  if (e != cudaSuccess) return e;
  const bool narrow = c.E <= 16;
  if (narrow && c.d % 8 == 0) {
    // about two CTAs per SM in all: each CTA loads its columns of W once, so
    // the rows of CTAs share that cost over as many tokens as possible
    const int gx = ceil_div(c.d, 1024);
    const dim3 grid((unsigned)gx, (unsigned)std::max(
                                      1, std::min(ceil_div(c.T, 16),
                                                  ceil_div(2 * device_sm_count(), gx))));
    e = c.E <= 8 ? launch_kernel(route_dx_narrow_kernel<8>, grid, 256, 0, s, 0, dlogits, W, c.T,
                                 c.d, c.E, dx)
                 : launch_kernel(route_dx_narrow_kernel<16>, grid, 256, 0, s, 0, dlogits, W, c.T,
                                 c.d, c.E, dx);
  } else {
    e = launch_kernel(route_dx_kernel,
                      dim3((unsigned)ceil_div(c.d, 256),
                           (unsigned)std::min(ceil_div(c.T, kTg), 65535)),
                      256, 0, s, 0, dlogits, W, c.T, c.d, c.E, dx);
  }
  if (e != cudaSuccess) return e;
  const int nchunks = route_backward_chunks(c.T, c.E);
  if (narrow && c.d % 8 == 0) {
    // E <= 8: 8 columns a thread; E <= 16: 4 (64 accumulators either way)
    const int cpt = c.E <= 8 ? 8 : 4;
    const dim3 ngrid((unsigned)ceil_div(c.d, 256 * cpt), (unsigned)nchunks);
    if (c.act_dtype == MOE_BF16) {
      const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
      e = c.E <= 8 ? launch_kernel(route_dw_narrow_kernel<__nv_bfloat16, 8, 8>, ngrid, 256, 0, s,
                                   0, xb, dlogits, c.T, c.d, c.E, nchunks, dw_part, dbias_part)
                   : launch_kernel(route_dw_narrow_kernel<__nv_bfloat16, 16, 4>, ngrid, 256, 0, s,
                                   0, xb, dlogits, c.T, c.d, c.E, nchunks, dw_part, dbias_part);
    } else {
      const float* xf = static_cast<const float*>(x);
      e = c.E <= 8 ? launch_kernel(route_dw_narrow_kernel<float, 8, 8>, ngrid, 256, 0, s, 0, xf,
                                   dlogits, c.T, c.d, c.E, nchunks, dw_part, dbias_part)
                   : launch_kernel(route_dw_narrow_kernel<float, 16, 4>, ngrid, 256, 0, s, 0, xf,
                                   dlogits, c.T, c.d, c.E, nchunks, dw_part, dbias_part);
    }
    if (e != cudaSuccess) return e;
    const int rblocks =
        (int)std::min<long long>((total + 255) / 256, (long long)device_sm_count() * 8);
    return launch_kernel(route_dw_reduce_kernel, rblocks, 256, 0, s, 0, dw_part, dbias_part, total,
                         c.E, nchunks, dW, dbias);
  }
  const dim3 grid((unsigned)ceil_div(c.d, kCt), (unsigned)nchunks);
  const size_t dsm = (size_t)kTs * c.E * sizeof(float);
  const int ept = c.E <= 8 ? 2 : c.E <= 16 ? 4 : c.E <= 32 ? 8 : c.E <= 64 ? 16 : c.E <= 128 ? 32 : 64;
  auto run = [&](auto kern) {
    cudaError_t r = ensure_smem_limit(reinterpret_cast<const void*>(kern), (int)dsm);
    if (r != cudaSuccess) return r;
    return launch_kernel(kern, grid, 256, dsm, s, 0, static_cast<const __nv_bfloat16*>(x),
                         dlogits, c.T, c.d, c.E, nchunks, dw_part, dbias_part);
  };
  auto runf = [&](auto kern) {
    cudaError_t r = ensure_smem_limit(reinterpret_cast<const void*>(kern), (int)dsm);
    if (r != cudaSuccess) return r;
    return launch_kernel(kern, grid, 256, dsm, s, 0, static_cast<const float*>(x), dlogits, c.T,
                         c.d, c.E, nchunks, dw_part, dbias_part);
  };
  if (c.act_dtype == MOE_BF16) {
    switch (ept) {
      case 2: e = run(route_dw_partial_kernel<__nv_bfloat16, 2>); break;
      case 4: e = run(route_dw_partial_kernel<__nv_bfloat16, 4>); break;
      case 8: e = run(route_dw_partial_kernel<__nv_bfloat16, 8>); break;
      case 16: e = run(route_dw_partial_kernel<__nv_bfloat16, 16>); break;
      case 32: e = run(route_dw_partial_kernel<__nv_bfloat16, 32>); break;
      default: e = run(route_dw_partial_kernel<__nv_bfloat16, 64>); break;
    }
  } else {
    switch (ept) {
      case 2: e = runf(route_dw_partial_kernel<float, 2>); break;
      case 4: e = runf(route_dw_partial_kernel<float, 4>); break;
      case 8: e = runf(route_dw_partial_kernel<float, 8>); break;
      case 16: e = runf(route_dw_partial_kernel<float, 16>); break;
      case 32: e = runf(route_dw_partial_kernel<float, 32>); break;
      default: e = runf(route_dw_partial_kernel<float, 64>); break;
    }
  }
  if (e != cudaSuccess) return e;
  const int rblocks = (int)std::min<long long>((total + 255) / 256, (long long)device_sm_count() * 8);
  return launch_kernel(route_dw_reduce_kernel, rblocks, 256, 0, s, 0, dw_part, dbias_part, total,
                       c.E, nchunks, dW, dbias);
}

}  // namespace moe
