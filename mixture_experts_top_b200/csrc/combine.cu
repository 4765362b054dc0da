// combine.cu - gate-weighted sum of each token's expert outputs.
//
// "Mixture-of-Experts Routing - LLM Internals" (mlgrind.dev), Algorithm 3:
//   y_t = sum_j gates[t, j] * expert_{indices[t, j]}(x_t).
// "Mixture of Experts: the Sparsely-Gated Layer" (paperfordummies.in),
// "Switch: top-1, one loss, and a rate limit": a dropped slot contributes 0.
//
// One warp per token, 16-byte vectors along the row; each output element is
// an fp32 fused multiply-add chain over j = 0..k-1 in that order (no atomics,
// so the result does not depend on scheduling), rounded once to the output
// dtype.  HBM bound: reads k rows, writes one.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

template <typename XT>
struct Vec16;

template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int kN = 8;
  __device__ static void fma_row(const void* p, float g, float (&acc)[8]) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] = fmaf(g, __uint_as_float(w[i] << 16), acc[2 * i]);
      acc[2 * i + 1] = fmaf(g, __uint_as_float(w[i] & 0xFFFF0000u), acc[2 * i + 1]);
    }
  }
  __device__ static void store(void* p, const float (&acc)[8]) {
    uint4 q;
    q.x = pack_bf16x2(acc[0], acc[1]);
    q.y = pack_bf16x2(acc[2], acc[3]);
    q.z = pack_bf16x2(acc[4], acc[5]);
    q.w = pack_bf16x2(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(p) = q;
  }
};

template <>
struct Vec16<float> {
  static constexpr int kN = 4;
  __device__ static void fma_row(const void* p, float g, float (&acc)[4]) {
    const float4 q = __ldg(reinterpret_cast<const float4*>(p));
    acc[0] = fmaf(g, q.x, acc[0]);
    acc[1] = fmaf(g, q.y, acc[1]);
    acc[2] = fmaf(g, q.z, acc[2]);
    acc[3] = fmaf(g, q.w, acc[3]);
  }
  __device__ static void store(void* p, const float (&acc)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  }
};

template <typename XT>
__global__ void __launch_bounds__(256)
    combine_kernel(const XT* __restrict__ y_perm, const int32_t* __restrict__ dest,
                   const float* __restrict__ gates, XT* __restrict__ out, int T, int k, int d_out) {
  constexpr int V = Vec16<XT>::kN;
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int nvec = d_out / V;
  for (int t = gw; t < T; t += nw) {
    int dl = -1;
    float gl = 0.f;
    if (lane < k) {
      dl = dest[(size_t)t * k + lane];
      gl = gates[(size_t)t * k + lane];
    }
    int dj[8];
    float gj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      dj[j] = __shfl_sync(0xffffffffu, dl, j);
      gj[j] = __shfl_sync(0xffffffffu, gl, j);
    }
    XT* orow = out + (size_t)t * d_out;
#pragma unroll 2
    for (int v = lane; v < nvec; v += 32) {
      float acc[V];
#pragma unroll
      for (int i = 0; i < V; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < k && dj[j] >= 0)
          Vec16<XT>::fma_row(y_perm + (size_t)dj[j] * d_out + (size_t)v * V, gj[j], acc);
      Vec16<XT>::store(orow + (size_t)v * V, acc);
    }
  }
}

}  // namespace

cudaError_t launch_combine(const moe_config_t& c, const void* y_perm, const int32_t* dest,
                           const float* gates, void* out, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  const int blocks = min(ceil_div(c.T, 8), device_sm_count() * 16);
  if (c.act_dtype == MOE_BF16)
    combine_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(y_perm), dest, gates, static_cast<__nv_bfloat16*>(out),
        c.T, c.top_k, c.d_out);
  else
    combine_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(y_perm), dest, gates,
                                                 static_cast<float*>(out), c.T, c.top_k, c.d_out);
  return cudaGetLastError();
}

}  // namespace moe
