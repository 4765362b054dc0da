// dispatch.cu - deterministic MoE dispatch: per-expert histogram, positions in
// token order, capacity, grouped layout, load-balancing loss, row gather.
//
// "Mixture-of-Experts Routing - LLM Internals" (mlgrind.dev), Algorithm 3-4
// and Follow-up; "Mixture of Experts: the Sparsely-Gated Layer"
// (paperfordummies.in), The code (`moe_forward`: tokens routed to an expert
// in token order, truncated to the capacity, first come first served) and
// "Switch: top-1, one loss, and a rate limit".
//
// Slots s = t*k + j are ranked in increasing s.  A slot's position p on its
// expert e is the number of earlier slots on e; it is kept iff p < cap, and
// then lands on grouped row offsets[e] + p, offsets being the exclusive scan
// of kept_e = min(count_e, cap).
//
// Two launches, no atomics on data, no scheduling-dependent order:
//   count   - one CTA per 256-token chunk; each warp ranks 32 tokens' slots
//             with __match_any_sync (peers with the same expert) against a
//             per-warp running histogram, then warps are offset by an
//             exclusive scan over warps.  Writes the chunk histogram and each
//             slot's rank inside its chunk.
//   scan    - in the last chunk's CTA to finish (a counter in the workspace
//             finds it; the result does not depend on which CTA it is): per
//             expert, exclusive scan of the chunk histograms over chunks
//             (chunk bases) and the total count; kept, offsets, f and aux = E
//             * sum f_e P_e (fp64, fixed-order butterfly).
//   scatter - one warp per token: dest, drop mask, perm_token, and the copy
//             of x[t] into every kept grouped row with 16-byte vectors (the
//             row's loads issued before the dependent index loads)
//             (skipped when x_perm is null: the up projection then gathers
//             the rows through perm_token itself).
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kCountWarps = kChunkTokens / 32;  // 8 warps, 32 tokens each
constexpr int kMaxE = 256;

__device__ __forceinline__ int warp_inclusive_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Arguments of the scan (one CTA): per expert, the exclusive scan of the
// chunk histograms over chunks (chunk bases) and the total; the capacity,
// offsets, f and aux; and, for a rank of a sharded batch, the earlier ranks'
// slots and the batch's P from the exchange records.
struct ScanArgs {
  const int32_t* chunk_counts;
  int nchunks, E, T, k;
  int64_t cap;
  const float* prob_mean;
  int32_t* chunk_base;
  int32_t* counts;
  int32_t* offsets;
  float* f;
  float* aux;
  const int32_t* records;
  int rank, world, T_global;
  int32_t* prefix;
  int32_t* err;
};

// The scan by the whole calling CTA (at least two warps).  The chunk
// histograms are read through L2: they may have been written by other CTAs
// of the same launch.
__device__ void dispatch_scan_body(const ScanArgs& a) {
  __shared__ int32_t s_counts[kMaxE];
  __shared__ int32_t s_prefix[kMaxE];   // slots of earlier ranks (sharded batch), else 0
  __shared__ int32_t s_total[kMaxE];    // slots of the whole batch
  __shared__ float s_P[kMaxE];          // P_e of the batch (sharded) or prob_mean
  const int E = a.E, nchunks = a.nchunks, T = a.T, k = a.k;
  const int64_t cap = a.cap;
  const int32_t* records = a.records;
  const int rank = a.rank, world = a.world, T_global = a.T_global;
  const int rec = 2 * E + 1;            // ints per exchange record
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  // A warp scans experts e0 + i * nwarps, i < 8, together: the 8 columns of
  // a 32-chunk block are loaded at once, then scanned one by one.
  for (int e0 = warp; e0 < E; e0 += 8 * nwarps) {
    int carry[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) carry[i] = 0;
    for (int c0 = 0; c0 < nchunks; c0 += 32) {
      const int c = c0 + lane;
      int v[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e0 + i * nwarps;
        v[i] = (c < nchunks && e < E) ? __ldcg(a.chunk_counts + (size_t)c * E + e) : 0;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int e = e0 + i * nwarps;
        if (e >= E) break;   // warp-uniform
        const int incl = warp_inclusive_scan(v[i]);
        if (c < nchunks) a.chunk_base[(size_t)c * E + e] = carry[i] + incl - v[i];
        carry[i] += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = e0 + i * nwarps;
      if (lane == 0 && e < E) s_counts[e] = carry[i];
    }
  }
  // Sharded batch: this rank's tokens follow those of ranks 0..rank-1 in
  // the batch order, so a slot's position on its expert is offset by their
  // slots on it; the capacity, f and aux are those of the whole batch, and
  // P_e is the token-weighted mean of the ranks' P_e, summed in fp64 in rank
  // order and rounded once to fp32.
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int pre = 0, tot = 0;
    float P = 0.f;
    if (records != nullptr) {
      double acc = 0.0;
      for (int r = 0; r < world; ++r) {
        const int32_t* rr = records + (size_t)r * rec;
        const int v = rr[e];
        if (r < rank) pre += v;
        tot += v;
        acc += (double)__int_as_float(rr[E + e]) * (double)rr[2 * E];
      }
      a.prefix[e] = pre;
      P = T_global > 0 ? (float)(acc / (double)T_global) : 0.f;
    } else {
      P = a.prob_mean[e];
    }
    s_prefix[e] = pre;
    s_total[e] = records != nullptr ? tot : 0;
    s_P[e] = P;
  }
  __syncthreads();
  if (records != nullptr) {
    for (int e = threadIdx.x; e < E; e += blockDim.x)
      if (records[(size_t)rank * rec + e] != s_counts[e]) report_error(a.err, kDevBadShard);
    if (threadIdx.x == 0) {
      long long tokens = 0;
      for (int r = 0; r < world; ++r) tokens += records[(size_t)r * rec + 2 * E];
      if (tokens != (long long)T_global || records[(size_t)rank * rec + 2 * E] != T)
        report_error(a.err, kDevBadShard);
    }
  }
  if (warp == 0) {
    int run = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int cnt = e < E ? s_counts[e] : 0;
      const int64_t room = cap < 0 ? (int64_t)cnt : cap - (int64_t)(e < E ? s_prefix[e] : 0);
      const int kept = room <= 0 ? 0 : (room < cnt ? (int)room : cnt);
      const int incl = warp_inclusive_scan(kept);
      if (e < E) {
        a.offsets[e] = run + incl - kept;
        a.counts[e] = cnt;
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) a.offsets[E] = run;
  } else if (warp == 1) {
    const bool sharded = records != nullptr;
    const double slots = (double)(sharded ? T_global : T) * (double)k;
    double acc = 0.0;
    for (int e = lane; e < E; e += 32) {
      const double fe = slots > 0.0 ? (double)(sharded ? s_total[e] : s_counts[e]) / slots : 0.0;
      a.f[e] = (float)fe;
      acc += fe * (double)s_P[e];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) a.aux[0] = (float)((double)E * acc);
  }
}

// The scan alone (no chunks to count: T = 0).
__global__ void __launch_bounds__(1024) dispatch_scan_kernel(const ScanArgs a) {
  pdl_wait_and_release();
  dispatch_scan_body(a);
}

__global__ void __launch_bounds__(kCountWarps * 32)
    dispatch_count_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                          int32_t* __restrict__ chunk_counts, int32_t* __restrict__ local_rank,
                          int32_t* err, const ScanArgs scan, unsigned* __restrict__ done) {
  pdl_wait_and_release();
  __shared__ int32_t whist[kCountWarps][kMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = lane; e < E; e += 32) whist[warp][e] = 0;
  __syncwarp();

  const int c = blockIdx.x;
  const int t0 = c * kChunkTokens + warp * 32;
  const int t1 = min(t0 + 32, T);
  const long s_begin = (long)t0 * k, s_end = (long)max(t1, t0) * k;
  const uint32_t lt = lanemask_lt();
  // The warp's 32 k slots, 32 at a time (k <= 8 rounds): every index load is
  // issued first; each slot's expert and rank stay in registers until the
  // ranks are final.
  int ev[8], rv[8];
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const long s = s_begin + 32 * it + lane;
    ev[it] = (it < k && s < s_end) ? idx[s] : -2;   // -2: no slot
  }
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    if (it >= k) break;
    int e = ev[it];
    if (e != -2 && (e < 0 || e >= E)) {
      report_error(err, kDevBadExpertIndex);
      e = -1;
    }
    if (e == -2) e = -1;
    ev[it] = e;
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    rv[it] = (e >= 0) ? whist[warp][e] + __popc(peers & lt) : 0;
    __syncwarp();
    if (e >= 0 && (peers & lt) == 0u) whist[warp][e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  // Exclusive scan over warps, per expert; the total is the chunk histogram.
  __shared__ int32_t wbase[kCountWarps][kMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kCountWarps; ++w) {
      wbase[w][e] = run;
      run += whist[w][e];
    }
    chunk_counts[(size_t)c * E + e] = run;
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    if (it >= k) break;
    const long s = s_begin + 32 * it + lane;
    if (s < s_end) local_rank[s] = rv[it] + (ev[it] >= 0 ? wbase[warp][ev[it]] : 0);
  }
  // With `done`, the last chunk's CTA to finish runs the scan (all chunk
  // histograms are complete and visible by then), and leaves `done` at 0.
  if (done != nullptr) {
    __threadfence();
    __syncthreads();
    __shared__ int s_last;
    if (threadIdx.x == 0) s_last = atomicAdd(done, 1u) == gridDim.x - 1u;
    __syncthreads();
    if (s_last) {
      __threadfence();
      dispatch_scan_body(scan);
      if (threadIdx.x == 0) atomicExch(done, 0u);
    }
  }
}

// PF: 16-byte vectors per lane loaded ahead, 32 * PF * 16 bytes of the row
// (the whole row where it fits: a deeper buffer for short rows only costs
// registers and occupancy); 0 for small batches, where the launch with fewer
// registers measured faster.
template <int ELEM, int PF>
__global__ void __launch_bounds__(256)
    dispatch_scatter_kernel(const uint8_t* __restrict__ x, const int32_t* __restrict__ idx,
                            int T, int k, int E, int d, int64_t cap,
                            const int32_t* __restrict__ chunk_base,
                            const int32_t* __restrict__ local_rank,
                            const int32_t* __restrict__ offsets, int32_t* __restrict__ dest,
                            int32_t* __restrict__ perm_token, uint8_t* __restrict__ drop_mask,
                            uint8_t* __restrict__ x_perm, const int32_t* __restrict__ prefix) {
  pdl_wait_and_release();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int nvec = d * ELEM / 16;  // 16-byte vectors per row
  const size_t row_bytes = (size_t)d * ELEM;
  for (int t = gw; t < T; t += nw) {
    // The row's first 32 * PF vectors are loaded before the index work, so
    // their latency overlaps the dependent index loads.
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * row_bytes);
    uint4 buf[PF > 0 ? PF : 1];
    if (x_perm != nullptr) {
#pragma unroll
      for (int i = 0; i < PF; ++i) {
        const int v = lane + 32 * i;
        if (v < nvec) buf[i] = __ldg(src + v);
      }
    }
    int my_dest = -1;
    if (lane < k) {
      const size_t s = (size_t)t * k + lane;
      const int e = idx[s];
      if (e >= 0 && e < E) {
        const int pos = chunk_base[(size_t)(t / kChunkTokens) * E + e] + local_rank[s];
        const int64_t gpos = (int64_t)pos + (prefix != nullptr ? prefix[e] : 0);
        if (cap < 0 || gpos < cap) my_dest = offsets[e] + pos;
      }
      dest[s] = my_dest;
      drop_mask[s] = my_dest < 0 ? 1 : 0;
      if (my_dest >= 0) perm_token[my_dest] = t;
    }
    if (x_perm == nullptr) continue;   // rows are gathered later, by the expert GEMM
    int dj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) dj[j] = __shfl_sync(0xffffffffu, my_dest, j);
#pragma unroll
    for (int i = 0; i < PF; ++i) {
      const int v = lane + 32 * i;
      if (v < nvec) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < k && dj[j] >= 0)
            reinterpret_cast<uint4*>(x_perm + (size_t)dj[j] * row_bytes)[v] = buf[i];
        }
      }
    }
#pragma unroll 4
    for (int v = lane + 32 * PF; v < nvec; v += 32) {
      const uint4 val = __ldg(src + v);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k && dj[j] >= 0)
          reinterpret_cast<uint4*>(x_perm + (size_t)dj[j] * row_bytes)[v] = val;
      }
    }
  }
}

}  // namespace

cudaError_t launch_dispatch(const moe_config_t& c, const void* x, const int32_t* idx,
                            const float* prob_mean, int32_t* counts, int32_t* offsets,
                            int32_t* dest, int32_t* perm_token, uint8_t* drop_mask, float* f,
                            float* aux, void* x_perm, int32_t* chunk_counts, int32_t* chunk_base,
                            int32_t* local_rank, int32_t* err, cudaStream_t s,
                            const ShardInfo* shard, int32_t* shard_prefix, unsigned* done) {
  const int nchunks = ceil_div(c.T, kChunkTokens);
  const int64_t cap = capacity_slots(c.capacity_factor, shard != nullptr ? shard->T_global : c.T,
                                     c.top_k, c.E);
  ScanArgs sa;
  sa.chunk_counts = chunk_counts;
  sa.nchunks = nchunks;
  sa.E = c.E;
  sa.T = c.T;
  sa.k = c.top_k;
  sa.cap = cap;
  sa.prob_mean = prob_mean;
  sa.chunk_base = chunk_base;
  sa.counts = counts;
  sa.offsets = offsets;
  sa.f = f;
  sa.aux = aux;
  sa.records = shard != nullptr ? shard->records : nullptr;
  sa.rank = shard != nullptr ? shard->rank : 0;
  sa.world = shard != nullptr ? shard->world : 1;
  sa.T_global = shard != nullptr ? shard->T_global : c.T;
  sa.prefix = shard != nullptr ? shard_prefix : nullptr;
  sa.err = err;
  cudaError_t e;
  if (nchunks > 0) {
    // count, with the scan in the last chunk's CTA when `done` is given
    e = launch_kernel(dispatch_count_kernel, nchunks, kCountWarps * 32, 0, s, 0, idx, c.T,
                      c.top_k, c.E, chunk_counts, local_rank, err, sa, done);
    if (e != cudaSuccess) return e;
  }
  if (nchunks == 0 || done == nullptr) {
    e = launch_kernel(dispatch_scan_kernel, 1, 1024, 0, s, 0, sa);
    if (e != cudaSuccess) return e;
  }
  if (c.T == 0) return cudaSuccess;
  const int elem = c.act_dtype == MOE_BF16 ? 2 : 4;
  const int blocks = min(ceil_div(c.T, 8), device_sm_count() * 16);
  // whole rows ahead up to 4 KiB (8 vectors a lane), else 8 KiB of the row;
  // none below 1024 tokens
  const bool deep = (size_t)c.d * elem > 32 * 8 * 16;
  auto kern = c.T < 1024
                  ? (elem == 2 ? dispatch_scatter_kernel<2, 0> : dispatch_scatter_kernel<4, 0>)
                  : elem == 2
                        ? (deep ? dispatch_scatter_kernel<2, 16> : dispatch_scatter_kernel<2, 8>)
                        : (deep ? dispatch_scatter_kernel<4, 16> : dispatch_scatter_kernel<4, 8>);
  return launch_kernel(kern, blocks,
                       256, 0, s, 0, static_cast<const uint8_t*>(x), idx, c.T, c.top_k, c.E, c.d,
                       cap, chunk_base, local_rank, offsets, dest, perm_token, drop_mask,
                       static_cast<uint8_t*>(x_perm),
                       shard != nullptr ? (const int32_t*)shard_prefix : nullptr);
}

// Slots per expert of these expert indices (the histogram every rank of a
// sharded batch contributes before the sharded dispatch); with prob_mean,
// the rank's whole exchange record: counts, the bits of prob_mean, T.
__global__ void __launch_bounds__(256)
    dispatch_total_kernel(const int32_t* __restrict__ chunk_counts, int nchunks, int E,
                          int32_t* __restrict__ counts, const float* __restrict__ prob_mean,
                          int T) {
  pdl_wait_and_release();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int v = 0;
    for (int c = 0; c < nchunks; ++c) v += chunk_counts[(size_t)c * E + e];
    counts[e] = v;
    if (prob_mean != nullptr) counts[E + e] = __float_as_int(prob_mean[e]);
  }
  if (prob_mean != nullptr && threadIdx.x == 0) counts[2 * E] = T;
}

cudaError_t launch_dispatch_count(const moe_config_t& c, const int32_t* idx, int32_t* counts,
                                  int32_t* chunk_counts, int32_t* local_rank, int32_t* err,
                                  cudaStream_t s, const float* prob_mean) {
  const int nchunks = ceil_div(c.T, kChunkTokens);
  if (nchunks > 0) {
    cudaError_t e = launch_kernel(dispatch_count_kernel, nchunks, kCountWarps * 32, 0, s, 0, idx,
                                  c.T, c.top_k, c.E, chunk_counts, local_rank, err, ScanArgs{},
                                  (unsigned*)nullptr);
    if (e != cudaSuccess) return e;
  }
  return launch_kernel(dispatch_total_kernel, 1, 256, 0, s, 0, chunk_counts, nchunks, c.E,
                       counts, prob_mean, c.T);
}

}  // namespace moe
