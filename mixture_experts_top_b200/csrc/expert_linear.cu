// expert_linear.cu - fp32 linear experts on grouped rows.
//
// "Mixture-of-Experts Routing - LLM Internals" (mlgrind.dev), Background and
// Inputs: expert_e(x) = x @ expert_weights[e], expert_weights (E, d, d_out).
// With a row permutation the grouped row r is read from token row perm[r]
// (the permute fused into the operand load).
//
// The fp32 results must hold to 1e-4 relative, which rules out TF32 tensor
// cores (10-bit mantissa); this is a plain fp32 FMA kernel.  Each thread
// produces one output element of one grouped row: it finds the row's expert
// by binary search over the offsets and runs the dot product in increasing
// input index.  A row range that is not a valid partition (offsets not
// monotone, or past the row buffer) is reported on the error word and left
// untouched.
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kMaxE = 256;

__global__ void __launch_bounds__(256)
    linear_expert_kernel(const float* __restrict__ x_perm, const int32_t* __restrict__ offsets,
                         const float* __restrict__ W, float* __restrict__ y_perm, int rows_max,
                         int E, int d, int d_out, int32_t* err,
                         const int32_t* __restrict__ perm, int T) {
  pdl_wait_and_release();
  __shared__ int32_t off[kMaxE + 1];
  __shared__ int ok;
  if (threadIdx.x == 0 && threadIdx.y == 0) ok = 1;
  __syncthreads();
  const int tid = threadIdx.y * blockDim.x + threadIdx.x;
  for (int e = tid; e <= E; e += blockDim.x * blockDim.y) off[e] = offsets[e];
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x * blockDim.y)
    if (off[e] > off[e + 1]) ok = 0;
  if (tid == 0 && (off[0] != 0 || off[E] > rows_max)) ok = 0;
  __syncthreads();
  if (!ok) {
    if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) report_error(err, kDevBadOffsets);
    return;
  }
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= d_out) return;
  for (int r = blockIdx.y * blockDim.y + threadIdx.y; r < off[E]; r += gridDim.y * blockDim.y) {
    int lo = 0, hi = E;  // off[lo] <= r < off[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (off[mid] <= r) lo = mid; else hi = mid;
    }
    int src = r;
    if (perm != nullptr) {
      src = perm[r];
      if (src < 0 || src >= T) {
        if (n == 0) report_error(err, kDevBadPerm);
        continue;
      }
    }
    const float* xr = x_perm + (size_t)src * d;
    const float* We = W + (size_t)lo * d * d_out + n;
    float acc = 0.f;
    for (int i = 0; i < d; ++i) acc = fmaf(xr[i], We[(size_t)i * d_out], acc);
    y_perm[(size_t)r * d_out + n] = acc;
  }
}

}  // namespace

cudaError_t launch_linear_expert(const moe_config_t& c, const float* x_perm,
                                 const int32_t* offsets, const float* W, float* y_perm,
                                 int32_t* err, cudaStream_t s, const int32_t* perm) {
  const int rows_max = c.T * c.top_k;
  if (rows_max == 0) return cudaSuccess;
  const dim3 block(32, 8);
  const dim3 grid(ceil_div(c.d_out, 32), min(ceil_div(rows_max, 8), 8192));
  return launch_kernel(linear_expert_kernel, grid, block, 0, s, 0, x_perm, offsets, W, y_perm,
                       rows_max, c.E, c.d, c.d_out, err, perm, c.T);
}

}  // namespace moe
