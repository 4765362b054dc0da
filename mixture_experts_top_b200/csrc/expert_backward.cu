// expert_backward.cu - the experts' backward around the grouped GEMMs of
// grouped_gemm_bwd.cu: the padded grouped layout, the fp32 linear expert's
// backward, and the sum of each token's row gradients.
//
// "Mixture-of-Experts Routing - LLM Internals" (mlgrind.dev), Algorithm 3:
// y_t = sum_j gates[t,j] expert_{idx[t,j]}(x_t), each expert run on its
// routed rows only.  The pages print no backward; these are its derivatives:
// a kept row's input gradient comes from its own expert, and a token's input
// gradient is the sum over its kept slots of its rows' gradients (plus the
// router's part).  An expert that receives no row gets a zero weight gradient
// ("Mixture of Experts: the Sparsely-Gated Layer", paperfordummies.in, Hot
// shards: an idle expert learns nothing).
//
//   pack            - padded layout for the bf16 GEMMs: expert e's rows start
//                     at p_e = sum over e' < e of ceil(rows_e' / 64) * 64;
//                     Xp = x_perm rows, dYp = dy_perm rows rounded to bf16,
//                     zero rows after each expert's rows
//   linear backward - fp32 experts (x @ W): dx_perm = dy_perm W_e^T and
//                     dW_e = x_e^T dy_e, fp32 FMA in fixed orders
//   permute backward- dx_t = dx_add_t + sum over kept j (increasing) of
//                     dx_perm[dest[t, j]], fp32, one warp per token
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kPadRows = kBwdPadRows;

// The rows of `offsets` into shared memory by one warp, checked to be a
// partition of [0, offsets[E]) with offsets[E] <= rows_max; if not, the
// error is recorded and every expert is given no rows.
__device__ bool load_offsets_warp(const int32_t* offsets, int E, int rows_max, int* row_off,
                                  int32_t* err) {
  const int lane = threadIdx.x & 31;
  for (int e = lane; e <= E; e += 32) row_off[e] = offsets[e];
  __syncwarp();
  bool ok = true;
  for (int e = lane; e < E; e += 32) ok = ok && (row_off[e] <= row_off[e + 1]);
  if (lane == 0) ok = ok && row_off[0] == 0 && row_off[E] <= rows_max;
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) {
    if (lane == 0 && blockIdx.x == 0) report_error(err, kDevBadOffsets);
    for (int e = lane; e <= E; e += 32) row_off[e] = 0;
  }
  __syncwarp();
  return ok;
}

// Checked offsets and padded offsets (E+1) into shared memory, by one warp.
__device__ bool padded_offsets_warp(const int32_t* offsets, int E, int rows_max, int* row_off,
                                    int* poff, int32_t* err) {
  const int lane = threadIdx.x & 31;
  const bool ok = load_offsets_warp(offsets, E, rows_max, row_off, err);
  int carry = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    const int pr = (ok && e < E) ? (row_off[e + 1] - row_off[e] + kPadRows - 1) / kPadRows * kPadRows
                                 : 0;
    int incl = pr;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (e < E) poff[e + 1] = carry + incl;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) poff[0] = 0;
  __syncwarp();
  return ok;
}

// One warp per padded row: Xp[p] = x_perm[src] (bf16) and dYp[p] =
// bf16(dy_perm[src]) for the expert's real rows, zeros for its padding.
// With saved pre-activations (pre != null: the training forward wrote the
// real rows), a padding row's pre-activations are zeroed too (pre_blocks
// blocks of kBwdPreBlock floats per row, block b at b * rows_pad rows).
__global__ void __launch_bounds__(256)
    pack_rows_kernel(const __nv_bfloat16* __restrict__ x_perm, const float* __restrict__ dy_perm,
                     const int32_t* __restrict__ offsets, int E, int d, int d_out, int rows_max,
                     int rows_pad, __nv_bfloat16* __restrict__ xp,
                     __nv_bfloat16* __restrict__ dyp, int32_t* err, float* __restrict__ pre,
                     int pre_blocks) {
  pdl_wait_and_release();
  __shared__ int row_off[257], poff[257];
  if (threadIdx.x < 32) padded_offsets_warp(offsets, E, rows_max, row_off, poff, err);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int total = min(poff[E], rows_pad);
  for (int p = gw; p < total; p += nw) {
    int lo = 0, hi = E;   // poff[lo] <= p < poff[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (poff[mid] <= p) lo = mid; else hi = mid;
    }
    const int local = p - poff[lo];
    const bool real = local < row_off[lo + 1] - row_off[lo];
    const size_t src = (size_t)(row_off[lo] + (real ? local : 0));
    const uint4* xs = reinterpret_cast<const uint4*>(x_perm + src * d);
    uint4* xd = reinterpret_cast<uint4*>(xp + (size_t)p * d);
    for (int v = lane; v < d / 8; v += 32) xd[v] = real ? __ldg(xs + v) : make_uint4(0, 0, 0, 0);
    const float4* ys = reinterpret_cast<const float4*>(dy_perm + src * d_out);
    uint4* yd = reinterpret_cast<uint4*>(dyp + (size_t)p * d_out);
    for (int v = lane; v < d_out / 8; v += 32) {
      if (real) {
        const float4 a = __ldg(ys + 2 * v), b = __ldg(ys + 2 * v + 1);
        yd[v] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y),
                           pack_bf16x2(b.z, b.w));
      } else {
        yd[v] = make_uint4(0, 0, 0, 0);
      }
    }
    if (pre != nullptr && !real)
      for (int b = 0; b < pre_blocks; ++b) {
        float4* pd = reinterpret_cast<float4*>(pre + ((size_t)b * rows_pad + p) * kBwdPreBlock);
        for (int v = lane; v < kBwdPreBlock / 4; v += 32) pd[v] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
  }
}

// fp32 linear experts, dx_perm[r, i] = sum_o dy[r, o] W_e[i, o]: one thread
// per (row, i), the sum over o in increasing order.
__global__ void __launch_bounds__(256)
    linear_dx_kernel(const float* __restrict__ dy, const int32_t* __restrict__ offsets,
                     const float* __restrict__ W, int E, int d, int d_out, int rows_max,
                     float* __restrict__ dx, int32_t* err) {
  pdl_wait_and_release();
  __shared__ int row_off[257];
  if (threadIdx.x < 32) load_offsets_warp(offsets, E, rows_max, row_off, err);
  __syncthreads();
  const int R = row_off[E];
  const long n = (long)R * d;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const int r = (int)(i / d), c = (int)(i % d);
    int lo = 0, hi = E;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (row_off[mid] <= r) lo = mid; else hi = mid;
    }
    const float* w = W + ((size_t)lo * d + c) * d_out;
    const float* g = dy + (size_t)r * d_out;
    float acc = 0.f;
    for (int o = 0; o < d_out; ++o) acc = fmaf(g[o], w[o], acc);
    dx[i] = acc;
  }
}

// fp32 linear experts, dW_e[i, o] = sum over the expert's rows r (increasing)
// of x[r, i] dy[r, o]: one thread per (e, i, o); zero for an expert without rows.
__global__ void __launch_bounds__(256)
    linear_dw_kernel(const float* __restrict__ x_perm, const float* __restrict__ dy,
                     const int32_t* __restrict__ offsets, int E, int d, int d_out, int rows_max,
                     float* __restrict__ dW, int32_t* err) {
  pdl_wait_and_release();
  __shared__ int row_off[257];
  if (threadIdx.x < 32) load_offsets_warp(offsets, E, rows_max, row_off, err);
  __syncthreads();
  const long n = (long)E * d * d_out;
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const int e = (int)(i / ((long)d * d_out));
    const int rem = (int)(i % ((long)d * d_out));
    const int c = rem / d_out, o = rem % d_out;
    float acc = 0.f;
    for (int r = row_off[e]; r < row_off[e + 1]; ++r)
      acc = fmaf(x_perm[(size_t)r * d + c], dy[(size_t)r * d_out + o], acc);
    dW[i] = acc;
  }
}

// dx[t] = (dx_add ? dx_add[t] : 0) + sum over kept j of dx_perm[dest[t, j]],
// j increasing, fp32; one warp per token, 4 columns per lane step.
__global__ void __launch_bounds__(256)
    permute_backward_kernel(const float* __restrict__ dx_perm, const int32_t* __restrict__ dest,
                            const float* __restrict__ dx_add, float* __restrict__ dx, int T, int k,
                            int d) {
  pdl_wait_and_release();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (int t = gw; t < T; t += nw) {
    const int dl = lane < k ? dest[(size_t)t * k + lane] : -1;
    int dj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) dj[j] = __shfl_sync(0xffffffffu, dl, j);
    for (int v = lane; v < d / 4; v += 32) {
      float4 acc = dx_add != nullptr ? reinterpret_cast<const float4*>(dx_add + (size_t)t * d)[v]
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k && dj[j] >= 0) {
          const float4 a = __ldg(reinterpret_cast<const float4*>(dx_perm + (size_t)dj[j] * d) + v);
          acc.x += a.x;
          acc.y += a.y;
          acc.z += a.z;
          acc.w += a.w;
        }
      }
      reinterpret_cast<float4*>(dx + (size_t)t * d)[v] = acc;
    }
  }
}

}  // namespace

ExpertBwdLayout expert_backward_layout(const moe_config_t& c) {
  ExpertBwdLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) / 256 * 256;
    return o;
  };
  L.ctrl = take(256);
  if (c.expert_kind != MOE_EXPERT_LINEAR) {
    const size_t Rp = (size_t)expert_backward_pad_rows(c.T * c.top_k, c.E);
    const size_t DHp = (size_t)ceil_div(c.d_hidden, 64) * 64;
    const size_t wide = (c.expert_kind == MOE_EXPERT_SWIGLU ? 2 : 1) * DHp;
    L.xp = take(Rp * (size_t)c.d * 2);
    L.dyp = take(Rp * (size_t)c.d_out * 2);
    // pre-activations in blocks of kBwdPreBlock hidden units (grouped_gemm_bwd.cu)
    const size_t pre_cols = (size_t)ceil_div(c.d_hidden, kBwdPreBlock) * kBwdPreBlock;
    L.pre = take(Rp * (c.expert_kind == MOE_EXPERT_SWIGLU ? 2 : 1) * pre_cols * 4);
    L.dab = take(Rp * wide * 2);
    L.hid = take(Rp * DHp * 2);
  }
  L.total = off;
  return L;
}

cudaError_t launch_expert_backward(const moe_config_t& c, const void* x_perm,
                                   const int32_t* offsets, const void* W_in, const void* W_up,
                                   const void* W_out, const float* dy_perm, float* dx_perm,
                                   float* dW_in, float* dW_up, float* dW_out, void* ws,
                                   cudaStream_t s, bool pre_saved) {
  const ExpertBwdLayout L = expert_backward_layout(c);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* err = reinterpret_cast<int32_t*>(base + L.ctrl);
  const int rows_max = c.T * c.top_k;
  const int sms = device_sm_count();
  if (c.expert_kind == MOE_EXPERT_LINEAR) {
    cudaError_t e = cudaSuccess;
    if (rows_max > 0) {
      const long n = (long)rows_max * c.d;
      e = launch_kernel(linear_dx_kernel, (int)std::min<long>((n + 255) / 256, (long)sms * 8), 256,
                        0, s, 0, dy_perm, offsets, static_cast<const float*>(W_in), c.E, c.d,
                        c.d_out, rows_max, dx_perm, err);
      if (e != cudaSuccess) return e;
    }
    const long nw = (long)c.E * c.d * c.d_out;
    return launch_kernel(linear_dw_kernel, (int)std::min<long>((nw + 255) / 256, (long)sms * 8),
                         256, 0, s, 0, static_cast<const float*>(x_perm), dy_perm, offsets, c.E,
                         c.d, c.d_out, rows_max, dW_in, err);
  }
  __nv_bfloat16* xp = reinterpret_cast<__nv_bfloat16*>(base + L.xp);
  __nv_bfloat16* dyp = reinterpret_cast<__nv_bfloat16*>(base + L.dyp);
  const int rows_pad = expert_backward_pad_rows(rows_max, c.E);
  if (rows_max > 0) {
    const int blocks = std::min(ceil_div(rows_pad, 8), sms * 8);
    const int pre_blocks = (c.expert_kind == MOE_EXPERT_SWIGLU ? 2 : 1) *
                           ceil_div(c.d_hidden, kBwdPreBlock);
    cudaError_t e = launch_kernel(pack_rows_kernel, blocks, 256, 0, s, 0,
                                  static_cast<const __nv_bfloat16*>(x_perm), dy_perm, offsets, c.E,
                                  c.d, c.d_out, rows_max, rows_pad, xp, dyp, err,
                                  pre_saved ? reinterpret_cast<float*>(base + L.pre) : nullptr,
                                  pre_blocks);
    if (e != cudaSuccess) return e;
  }
  return launch_expert_backward_gemms(
      c, offsets, xp, dyp, static_cast<const __nv_bfloat16*>(W_in),
      static_cast<const __nv_bfloat16*>(W_up), static_cast<const __nv_bfloat16*>(W_out),
      reinterpret_cast<float*>(base + L.pre), reinterpret_cast<__nv_bfloat16*>(base + L.dab),
      reinterpret_cast<__nv_bfloat16*>(base + L.hid), dx_perm, dW_in, dW_up, dW_out, err, s,
      pre_saved);
}

cudaError_t launch_permute_backward(const moe_config_t& c, const float* dx_perm,
                                    const int32_t* dest, const float* dx_add, float* dx,
                                    cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  const int blocks = std::min(ceil_div(c.T, 8), device_sm_count() * 16);
  return launch_kernel(permute_backward_kernel, blocks, 256, 0, s, 0, dx_perm, dest, dx_add, dx,
                       c.T, c.top_k, c.d);
}

}  // namespace moe
