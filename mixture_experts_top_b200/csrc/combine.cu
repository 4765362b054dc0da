// combine.cu - gate-weighted sum of each token's expert outputs.
//
// "Mixture-of-Experts Routing - LLM Internals" (mlgrind.dev), Algorithm 3:
//   y_t = sum_j gates[t, j] * expert_{indices[t, j]}(x_t).
// "Mixture of Experts: the Sparsely-Gated Layer" (paperfordummies.in),
// "Switch: top-1, one loss, and a rate limit": a dropped slot contributes 0.
//
// The expert rows arrive in fp32 (the experts' unrounded outputs).  One warp
// per token, 8 columns per lane step (two 16-byte loads per expert row); each
// output element is an fp32 fused multiply-add chain over j = 0..k-1 in that
// order (no atomics, so the result does not depend on scheduling), rounded
// once to the layer's dtype.  HBM bound: reads k rows, writes one.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

// Stores 8 fp32 accumulators as 8 output elements.
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&a)[8]) {
  *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(a[0], a[1]), pack_bf16x2(a[2], a[3]),
                                            pack_bf16x2(a[4], a[5]), pack_bf16x2(a[6], a[7]));
}
__device__ __forceinline__ void store8(float* p, const float (&a)[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(a[0], a[1], a[2], a[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(a[4], a[5], a[6], a[7]);
}

// y_perm rows are the experts' fp32 outputs; OutT is the layer's dtype.
template <typename OutT>
__global__ void __launch_bounds__(256)
    combine_kernel(const float* __restrict__ y_perm, const int32_t* __restrict__ dest,
                   const float* __restrict__ gates, OutT* __restrict__ out, int T, int k,
                   int d_out) {
  pdl_wait_and_release();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int nvec = d_out / 8;  // 8 columns per lane step
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
    OutT* orow = out + (size_t)t * d_out;
#pragma unroll 2
    for (int v = lane; v < nvec; v += 32) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k && dj[j] >= 0) {
          const float4* src = reinterpret_cast<const float4*>(y_perm + (size_t)dj[j] * d_out) + 2 * v;
          const float4 a = __ldg(src), b = __ldg(src + 1);
          acc[0] = fmaf(gj[j], a.x, acc[0]);
          acc[1] = fmaf(gj[j], a.y, acc[1]);
          acc[2] = fmaf(gj[j], a.z, acc[2]);
          acc[3] = fmaf(gj[j], a.w, acc[3]);
          acc[4] = fmaf(gj[j], b.x, acc[4]);
          acc[5] = fmaf(gj[j], b.y, acc[5]);
          acc[6] = fmaf(gj[j], b.z, acc[6]);
          acc[7] = fmaf(gj[j], b.w, acc[7]);
        }
      }
      store8(orow + (size_t)v * 8, acc);
    }
  }
}

}  // namespace

cudaError_t launch_combine(const moe_config_t& c, const float* y_perm, const int32_t* dest,
                           const float* gates, void* out, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  const int blocks = min(ceil_div(c.T, 8), device_sm_count() * 16);
  if (c.act_dtype == MOE_BF16)
    return launch_kernel(combine_kernel<__nv_bfloat16>, blocks, 256, 0, s, 0, y_perm, dest, gates,
                         static_cast<__nv_bfloat16*>(out), c.T, c.top_k, c.d_out);
  return launch_kernel(combine_kernel<float>, blocks, 256, 0, s, 0, y_perm, dest, gates,
                       static_cast<float*>(out), c.T, c.top_k, c.d_out);
}

}  // namespace moe
