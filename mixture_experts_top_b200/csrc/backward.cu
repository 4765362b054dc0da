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
// logit gradient one warp per token; dx one thread per 4 output columns, the
// E terms in order; dW and dbias as per-chunk partial sums over token chunks,
// then the chunks added in order.  Everything here is bound by HBM or by
// launch latency.
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

// dx[t, c..c+3] = sum_e dL[t, e] W[c..c+3, e], e in increasing order.
__global__ void __launch_bounds__(256)
    route_dx_kernel(const float* __restrict__ dlogits, const float* __restrict__ W, int T, int d,
                    int E, float* __restrict__ dx) {
  pdl_wait_and_release();
  const long long n4 = (long long)T * (d / 4);
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const long long t = i / (d / 4);
    const int c = (int)(i - t * (d / 4)) * 4;
    const float* dl = dlogits + t * E;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int e = 0; e < E; ++e) {
      const float g = dl[e];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] = fmaf(g, W[(size_t)(c + u) * E + e], acc[u]);
    }
    *reinterpret_cast<float4*>(dx + t * d + c) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  }
}

constexpr int kDwOuts = 8;        // (c, e) outputs per thread
constexpr int kDwThreads = 256;

// Partial dW and dbias over one chunk of tokens: CTA (tile, chunk) owns the
// outputs o = tile * 2048 + [0, 2048) of the flattened (d, E) dW, i.e.
// c = o / E, e = o % E, and sums its tokens in increasing order.
template <typename XT>
__global__ void __launch_bounds__(kDwThreads)
    route_dw_partial_kernel(const XT* __restrict__ x, const float* __restrict__ dlogits, int T,
                            int d, int E, int nchunks, float* __restrict__ dw_part,
                            float* __restrict__ dbias_part) {
  pdl_wait_and_release();
  const int chunk = blockIdx.y;
  const int t0 = (int)((long long)T * chunk / nchunks);
  const int t1 = (int)((long long)T * (chunk + 1) / nchunks);
  const long long total = (long long)d * E;
  long long o[kDwOuts];
  int cc[kDwOuts], ee[kDwOuts];
  float acc[kDwOuts];
#pragma unroll
  for (int i = 0; i < kDwOuts; ++i) {
    o[i] = (long long)blockIdx.x * (kDwThreads * kDwOuts) + threadIdx.x + i * kDwThreads;
    cc[i] = (int)(o[i] / E);
    ee[i] = (int)(o[i] - (long long)cc[i] * E);
    acc[i] = 0.f;
  }
  float bacc = 0.f;                          // dbias[threadIdx.x], tile 0 only
  const bool do_bias = blockIdx.x == 0 && (int)threadIdx.x < E;
  for (int t = t0; t < t1; ++t) {
    const XT* xr = x + (size_t)t * d;
    const float* dl = dlogits + (size_t)t * E;
#pragma unroll
    for (int i = 0; i < kDwOuts; ++i)
      if (o[i] < total) acc[i] = fmaf(static_cast<float>(xr[cc[i]]), dl[ee[i]], acc[i]);
    if (do_bias) bacc += dl[threadIdx.x];
  }
#pragma unroll
  for (int i = 0; i < kDwOuts; ++i)
    if (o[i] < total) dw_part[(size_t)chunk * total + o[i]] = acc[i];
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
    float v = 0.f;
    for (int c = 0; c < nchunks; ++c) v += dw_part[(size_t)c * total + i];
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

int route_backward_chunks(int T) { return std::max(1, std::min(16, ceil_div(T, 128))); }

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
  const long long n4 = (long long)c.T * (c.d / 4);
  const int xblocks = (int)std::min<long long>((n4 + 255) / 256, (long long)device_sm_count() * 16);
  e = launch_kernel(route_dx_kernel, xblocks, 256, 0, s, 0, dlogits, W, c.T, c.d, c.E, dx);
  if (e != cudaSuccess) return e;
  const int nchunks = route_backward_chunks(c.T);
  const dim3 grid((unsigned)((total + kDwThreads * kDwOuts - 1) / (kDwThreads * kDwOuts)),
                  (unsigned)nchunks);
  if (c.act_dtype == MOE_BF16)
    e = launch_kernel(route_dw_partial_kernel<__nv_bfloat16>, grid, kDwThreads, 0, s, 0,
                      static_cast<const __nv_bfloat16*>(x), dlogits, c.T, c.d, c.E, nchunks,
                      dw_part, dbias_part);
  else
    e = launch_kernel(route_dw_partial_kernel<float>, grid, kDwThreads, 0, s, 0,
                      static_cast<const float*>(x), dlogits, c.T, c.d, c.E, nchunks, dw_part,
                      dbias_part);
  if (e != cudaSuccess) return e;
  const int rblocks = (int)std::min<long long>((total + 255) / 256, (long long)device_sm_count() * 8);
  return launch_kernel(route_dw_reduce_kernel, rblocks, 256, 0, s, 0, dw_part, dbias_part, total,
                       c.E, nchunks, dW, dbias);
}

}  // namespace moe
