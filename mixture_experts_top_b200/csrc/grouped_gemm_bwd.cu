// grouped_gemm_bwd.cu - the experts' backward on Blackwell tensor cores
// (tcgen05 + tensor memory): four grouped bf16 GEMMs with fp32 accumulation.
//
// The pages print no backward; these are the derivatives of the experts of
// "Mixture-of-Experts Routing - LLM Internals" (mlgrind.dev), Algorithm 3
// (each expert runs only on its routed rows), with the ReLU expert of
// "Mixture of Experts: the Sparsely-Gated Layer" (paperfordummies.in), The
// code, `expert_forward`, and the SwiGLU expert the pages name (silu(x Wg) *
// (x Wu)) Wd.  For the rows X of one expert, the gradient dY of its outputs
// and A = X W_in (B = X W_up), H the hidden activation:
//   dH = dY W_out^T
//   ReLU:   dA = dH * [A > 0],                  H = relu(A)
//   SwiGLU: s = sigmoid(A), dA = dH * B * s (1 + A (1 - s)), dB = dH * A s,
//           H = A s B
//   dX = dA W_in^T (+ dB W_up^T)
//   dW_out = H^T dY, dW_in = X^T dA, dW_up = X^T dB
//
// Every operand works on a padded grouped layout: expert e owns padded rows
// [p_e, p_e+1), p_e = sum over e' < e of ceil(rows_e' / 128) * 128, its rows
// first and zero rows after them.  No tile then straddles two experts, and
// the zero rows add nothing to any product (their pre-activations, dH, dA,
// dB and H are zero too).  The four GEMMs (one kernel, the stage selected by
// a template argument):
//   kPre   (M rows, N hidden, K d)      pre = Xp [W_in | W_up]: A and B of
//          the forward, recomputed, stored fp32 as [A | B] per row
//   kDH    (M rows, N hidden, K d_out)  dH = dYp W_out^T; the epilogue reads
//          the row's pre-activations and writes dAB = [dA | dB] and H (bf16)
//   kDX    (M rows, N d, K 2 hidden)    dX = dAB [W_in | W_up]^T, written as
//          fp32 rows of the unpadded grouped layout
//   kWgrad (M weight rows, N weight columns, K = the expert's padded rows)
//          dW_out = H^T dYp, dW_in = Xp^T dA, dW_up = Xp^T dB (fp32)
// Operand majors: kPre A K-major / B N-major (the weights as stored);
// kDH, kDX A K-major / B K-major (W^T: the stored weights read along their
// rows); kWgrad A M-major / B N-major (both activations, K running down their
// rows).  All are staged by TMA with 128-byte swizzle; the tensor core reads
// either major from shared memory, so no operand is transposed in memory.
//
// B200 design as in grouped_gemm.cu's single-CTA kernel: persistent, one CTA
// per SM, warp 0 TMA producer, warp 1 MMA issuer and tensor-memory owner,
// warps 2-5 epilogue; 128 x 256 tiles, k block 64, a 4-stage ring of 48 KiB,
// two 256-column accumulators; every wait bounded (the error word records a
// timeout, copies and MMAs are drained and tensor memory is freed).
#include <cudaTypedefs.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int BM = kBwdPadRows;   // tile rows = the padding of each expert's rows
constexpr int BK = 64;
constexpr int BN = 256;
constexpr int UK = 16;
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK * 2;          // 16 KiB
constexpr int BOX64 = 64 * BK * 2;            // one 64 x 64 box: 8 KiB
constexpr int B_STAGE = BN * BK * 2;          // 32 KiB
constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 2 * BN;
constexpr int MAX_E = 256;
constexpr int AUX_BYTES = 6144;               // barriers, tmem address, offsets, tile table
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + AUX_BYTES;

enum BwdStage { kPre = 0, kDH = 1, kDX = 2, kWgrad = 3 };

// Instruction descriptor, kind::f16 (bf16 x bf16 -> fp32), M = 128, N = 256:
// D fp32 (bit 4), A bf16 (7-9 = 1), B bf16 (10-12 = 1), A major at bit 15 and
// B major at bit 16 (0 = K-major, 1 = MN-major), N >> 3 at 17, M >> 4 at 24.
template <int STAGE>
struct Idesc {
  static constexpr uint32_t a_mn = STAGE == kWgrad ? 1u : 0u;
  static constexpr uint32_t b_mn = (STAGE == kPre || STAGE == kWgrad) ? 1u : 0u;
  static constexpr uint32_t value = (1u << 4) | (1u << 7) | (1u << 10) | (a_mn << 15) |
                                    (b_mn << 16) | ((uint32_t)(BN >> 3) << 17) |
                                    ((uint32_t)(BM >> 4) << 24);
};

// Shared-memory matrix descriptors, 128-byte swizzle, version 1 (bit 46),
// swizzle mode 2 (bits 61-63).
// K-major: rows of 128 bytes (64 k), 8-row groups 1024 bytes apart (stride
// byte offset); the leading byte offset is unused (16 bytes).  One UK step
// advances the start address by 32 bytes.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// MN-major: boxes of 64 MN elements (128 bytes) x 64 k rows; boxes along MN
// are BOX64 bytes apart (leading byte offset), 8-k-row groups 1024 bytes
// apart (stride byte offset).  One UK step advances 16 k rows = 2048 bytes.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(BOX64 >> 4) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

struct BwdArgs {
  const int32_t* offsets;   // (E+1) grouped rows of each expert (unpadded)
  int32_t* err;
  int E, K, N;              // this stage's contraction length and output width
  int swiglu;
  int d, DH, DHp, d_out;    // DHp: DH rounded up to 64
  int n_tiles;              // row-grouped stages: output-column blocks
  int rows_max;             // rows of the unpadded grouped buffers (T * top_k)
  float* pre;               // (Rp, (1 + swiglu) DHp) fp32: [A | B] pre-activations
  __nv_bfloat16* dab;       // (Rp, (1 + swiglu) DHp): [dA | dB]
  __nv_bfloat16* hid;       // (Rp, DHp): H
  float* dx;                // (R, d): unpadded grouped rows
  float* dw0;               // kWgrad: dW_out (E, DH, d_out)
  float* dw1;               //         dW_in  (E, d, DH)
  float* dw2;               //         dW_up  (E, d, DH) (SwiGLU)
};

// Weight-gradient problems of kWgrad: p = 0 dW_out (M DH, N d_out), p = 1
// dW_in (M d, N DH), p = 2 dW_up (M d, N DH; SwiGLU only).
__device__ __forceinline__ void wgrad_shape(const BwdArgs& g, int p, int& M, int& N) {
  M = p == 0 ? g.DH : g.d;
  N = p == 0 ? g.d_out : g.DH;
}

struct Tile {
  int e, m0, n0, p, kb0, nkb;   // kb0/nkb: first k block and count (kWgrad)
  int rows;                     // row-grouped stages: the expert's real rows
  int pr0;                      // row-grouped: first padded row of the expert
};

__device__ __forceinline__ float sigmoid_f(float a) { return 1.0f / (1.0f + __expf(-a)); }

template <int STAGE>
__device__ __forceinline__ Tile decode(int tile, const int* prefix, const int* poff,
                                       const int* row_off, const BwdArgs& g) {
  Tile t{};
  if (STAGE != kWgrad) {
    int lo = 0, hi = g.E;  // prefix[lo] <= tile < prefix[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= tile) lo = mid; else hi = mid;
    }
    const int local = tile - prefix[lo];
    const int mt = (poff[lo + 1] - poff[lo]) / BM;
    t.e = lo;
    t.n0 = (local / mt) * (STAGE == kPre ? (g.swiglu ? BN / 2 : BN) : BN);
    t.m0 = poff[lo] + (local % mt) * BM;
    t.rows = row_off[lo + 1] - row_off[lo];
    t.pr0 = poff[lo];
    t.p = 0;
    t.kb0 = 0;
    t.nkb = (g.K + BK - 1) / BK;
  } else {
    // problems in order p = 0, 1, 2; within one: expert, m block, n block
    int p = 0, base = 0;
    for (; p < 3; ++p) {
      int M, N;
      wgrad_shape(g, p, M, N);
      const int cnt = g.E * ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
      if (tile < base + cnt) break;
      base += cnt;
    }
    int M, N;
    wgrad_shape(g, p, M, N);
    const int mt = (M + BM - 1) / BM, nt = (N + BN - 1) / BN;
    const int local = tile - base;
    t.p = p;
    t.e = local / (mt * nt);
    const int rem = local % (mt * nt);
    t.m0 = (rem / nt) * BM;
    t.n0 = (rem % nt) * BN;
    t.kb0 = poff[t.e] / BK;
    t.nkb = (poff[t.e + 1] - poff[t.e]) / BK;
  }
  return t;
}

template <int STAGE>
__device__ __forceinline__ void epilogue_tile(uint32_t tacc, const Tile& t, int row,
                                              const BwdArgs& g) {
  if (STAGE == kPre) {
    // row: padded row; columns [n0, n0 + 128) gate / up (SwiGLU) or
    // [n0, n0 + 256) (ReLU) of the pre-activations, kept in fp32.
    const size_t ld = (size_t)(g.swiglu ? 2 : 1) * g.DHp;
    float* prow = g.pre + (size_t)(t.m0 + row) * ld;
    const int halves = g.swiglu ? 2 : 1;
    const int per = BN / halves;
#pragma unroll 1
    for (int h = 0; h < halves; ++h) {
#pragma unroll 1
      for (int cc = 0; cc < per; cc += 32) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tacc + (uint32_t)(h * per + cc), r);
        tmem_ld_wait();
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const int col = t.n0 + cc + v * 4;
          if (col < g.DHp)
            *reinterpret_cast<uint4*>(prow + (size_t)h * g.DHp + col) =
                make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
        }
      }
    }
  } else if (STAGE == kDH) {
    const size_t ld = (size_t)(g.swiglu ? 2 : 1) * g.DHp;
    const size_t r = (size_t)(t.m0 + row);
    const float* prow = g.pre + r * ld;
    __nv_bfloat16* drow = g.dab + r * ld;
    __nv_bfloat16* hrow = g.hid + r * (size_t)g.DHp;
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 32) {
      uint32_t acc[32];
      tmem_ld_32x32b_x32(tacc + (uint32_t)cc, acc);
      tmem_ld_wait();
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int col = t.n0 + cc + v * 8;
        if (col >= g.DHp) continue;
        float av[8], bv[8];
        {
          const float4 a0 = *reinterpret_cast<const float4*>(prow + col);
          const float4 a1 = *reinterpret_cast<const float4*>(prow + col + 4);
          av[0] = a0.x; av[1] = a0.y; av[2] = a0.z; av[3] = a0.w;
          av[4] = a1.x; av[5] = a1.y; av[6] = a1.z; av[7] = a1.w;
          if (g.swiglu) {
            const float4 b0 = *reinterpret_cast<const float4*>(prow + g.DHp + col);
            const float4 b1 = *reinterpret_cast<const float4*>(prow + g.DHp + col + 4);
            bv[0] = b0.x; bv[1] = b0.y; bv[2] = b0.z; bv[3] = b0.w;
            bv[4] = b1.x; bv[5] = b1.y; bv[6] = b1.z; bv[7] = b1.w;
          }
        }
        uint32_t da[4], db[4], hh[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float dA2[2], dB2[2], H2[2];
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const float a = av[2 * i + hf];
            const float dh = __uint_as_float(acc[v * 8 + 2 * i + hf]);
            if (g.swiglu) {
              const float b = bv[2 * i + hf];
              const float s = sigmoid_f(a);
              const float silu = a * s;
              dA2[hf] = dh * b * (s * (1.0f + a * (1.0f - s)));
              dB2[hf] = dh * silu;
              H2[hf] = silu * b;
            } else {
              dA2[hf] = a > 0.0f ? dh : 0.0f;
              dB2[hf] = 0.0f;
              H2[hf] = fmaxf(a, 0.0f);
            }
          }
          da[i] = pack_bf16x2(dA2[0], dA2[1]);
          db[i] = pack_bf16x2(dB2[0], dB2[1]);
          hh[i] = pack_bf16x2(H2[0], H2[1]);
        }
        *reinterpret_cast<uint4*>(drow + col) = make_uint4(da[0], da[1], da[2], da[3]);
        if (g.swiglu)
          *reinterpret_cast<uint4*>(drow + g.DHp + col) = make_uint4(db[0], db[1], db[2], db[3]);
        *reinterpret_cast<uint4*>(hrow + col) = make_uint4(hh[0], hh[1], hh[2], hh[3]);
      }
    }
  } else if (STAGE == kDX) {
    // padded row -> the expert's unpadded grouped row (zero rows are skipped)
    const int local = t.m0 + row - t.pr0;
    const bool valid = local < t.rows;
    float* orow = g.dx + (size_t)(g.offsets[t.e] + (valid ? local : 0)) * g.d;
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tacc + (uint32_t)cc, r);
      tmem_ld_wait();
      if (valid) {
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const int col = t.n0 + cc + v * 4;
          if (col < g.d)
            *reinterpret_cast<uint4*>(orow + col) =
                make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
        }
      }
    }
  } else {
    int M, N;
    wgrad_shape(g, t.p, M, N);
    float* dw = t.p == 0 ? g.dw0 : (t.p == 1 ? g.dw1 : g.dw2);
    const int m = t.m0 + row;
    const bool valid = m < M;
    float* orow = dw + ((size_t)t.e * M + (valid ? m : 0)) * N;
#pragma unroll 1
    for (int cc = 0; cc < BN; cc += 32) {
      uint32_t r[32];
      if (t.nkb > 0) {
        tmem_ld_32x32b_x32(tacc + (uint32_t)cc, r);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = 0u;   // an expert without rows: zero gradient
      }
      if (valid) {
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const int col = t.n0 + cc + v * 4;
          if (col < N)
            *reinterpret_cast<uint4*>(orow + col) =
                make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
        }
      }
    }
  }
}

// Tensor maps of one stage: A, B0, B1 (the second weight of SwiGLU, or the
// second activation map), and A1 (kWgrad: the second A source).
template <int STAGE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                    const BwdArgs g) {
  pdl_wait_and_release();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* drain_bar = tempty_bar + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain_bar + 1);
  int* tile_prefix = reinterpret_cast<int*>(tmem_holder + 4);   // MAX_E + 1
  int* poff = tile_prefix + (MAX_E + 1);                         // MAX_E + 1
  int* row_off = poff + (MAX_E + 1);                             // MAX_E + 1

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = g.E;

  if (warp == 0) {
    // Row offsets, padded offsets (rows per expert rounded up to BM) and,
    // for the row-grouped stages, the tile prefix (expert-major).
    for (int e = lane; e <= E; e += 32) row_off[e] = g.offsets[e];
    __syncwarp();
    bool ok = true;
    for (int e = lane; e < E; e += 32) ok = ok && (row_off[e] <= row_off[e + 1]);
    if (lane == 0) ok = ok && row_off[0] == 0 && row_off[E] <= g.rows_max;
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0 && blockIdx.x == 0) report_error(g.err, kDevBadOffsets);
    int carry_rows = 0, carry_tiles = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int pr = (ok && e < E) ? (row_off[e + 1] - row_off[e] + BM - 1) / BM * BM : 0;
      int incl = pr;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      if (e < E) {
        poff[e + 1] = carry_rows + incl;
        tile_prefix[e + 1] = carry_tiles + (incl / BM) * g.n_tiles;
      }
      carry_rows += __shfl_sync(0xffffffffu, incl, 31);
      carry_tiles = carry_rows / BM * g.n_tiles;
    }
    if (lane == 0) {
      poff[0] = 0;
      tile_prefix[0] = 0;
      tma_prefetch_map(&tmA);
      tma_prefetch_map(&tmA1);
      tma_prefetch_map(&tmB0);
      tma_prefetch_map(&tmB1);
    }
  } else if (warp == 1) {
    tmem_alloc(tmem_holder, TMEM_COLS);
    tmem_relinquish();
  } else if (warp == 2 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 128);
    }
    mbar_init(drain_bar, 1);
    fence_mbar_init();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;
  int total_tiles;
  if (STAGE == kWgrad) {
    total_tiles = 0;
    for (int p = 0; p < (g.swiglu ? 3 : 2); ++p) {
      int M, N;
      wgrad_shape(g, p, M, N);
      total_tiles += E * ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
    }
  } else {
    total_tiles = tile_prefix[E];
  }

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, last_phase = 0;
    bool alive = true;
    const uint64_t keep = l2_policy_evict_last(), stream = l2_policy_evict_normal();
    for (int tile = blockIdx.x; tile < total_tiles && alive; tile += gridDim.x) {
      const Tile t = decode<STAGE>(tile, tile_prefix, poff, row_off, g);
      for (int kb = 0; kb < t.nkb; ++kb) {
        uint8_t* sa = smem + stage * STAGE_BYTES;
        uint8_t* sb = sa + A_STAGE;
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) {
          report_error(g.err, kDevTimeoutProducer);
          alive = false;
          break;
        }
        mbar_arrive_expect_tx(&full_bar[stage], STAGE_BYTES);
        const int k0 = (t.kb0 + kb) * BK;
        if (STAGE == kPre) {
          tma_load_2d_hint(sa, &tmA, &full_bar[stage], k0, t.m0, keep);
          if (g.swiglu) {
            tma_load_3d_hint(sb, &tmB0, &full_bar[stage], t.n0, k0, t.e, stream);
            tma_load_3d_hint(sb + BOX64, &tmB0, &full_bar[stage], t.n0 + 64, k0, t.e, stream);
            tma_load_3d_hint(sb + 2 * BOX64, &tmB1, &full_bar[stage], t.n0, k0, t.e, stream);
            tma_load_3d_hint(sb + 3 * BOX64, &tmB1, &full_bar[stage], t.n0 + 64, k0, t.e, stream);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
              tma_load_3d_hint(sb + i * BOX64, &tmB0, &full_bar[stage], t.n0 + 64 * i, k0, t.e,
                               stream);
          }
        } else if (STAGE == kDH) {
          // A: dYp rows; B: W_out[e] read along its rows (K-major), 256 rows
          tma_load_2d_hint(sa, &tmA, &full_bar[stage], k0, t.m0, keep);
          tma_load_3d_hint(sb, &tmB0, &full_bar[stage], k0, t.n0, t.e, stream);
        } else if (STAGE == kDX) {
          // A: dAB rows; B: W_in[e] for k < DHp, W_up[e] beyond (K-major)
          tma_load_2d_hint(sa, &tmA, &full_bar[stage], k0, t.m0, keep);
          if (k0 < g.DHp)
            tma_load_3d_hint(sb, &tmB0, &full_bar[stage], k0, t.n0, t.e, stream);
          else
            tma_load_3d_hint(sb, &tmB1, &full_bar[stage], k0 - g.DHp, t.n0, t.e, stream);
        } else {
          // A (M-major): H (p = 0) or Xp (p >= 1), two 64-column boxes;
          // B (N-major): dYp (p = 0) or dAB columns (dA: p = 1, dB: p = 2)
          const CUtensorMap* am = t.p == 0 ? &tmA : &tmA1;
          const CUtensorMap* bm = t.p == 0 ? &tmB0 : &tmB1;
          const int bcol = t.p == 2 ? g.DHp : 0;
          tma_load_2d_hint(sa, am, &full_bar[stage], t.m0, k0, stream);
          tma_load_2d_hint(sa + BOX64, am, &full_bar[stage], t.m0 + 64, k0, stream);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            tma_load_2d_hint(sb + i * BOX64, bm, &full_bar[stage], bcol + t.n0 + 64 * i, k0,
                             stream);
        }
        issued_mask |= 1u << stage;
        last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    for (int s = 0; s < STAGES; ++s)
      if ((issued_mask >> s) & 1u)
        if (!mbar_wait(&full_bar[s], (last_phase >> s) & 1u)) report_error(g.err, kDevTimeoutDrain);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------ MMA issuer
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool alive = true;
    for (int tile = blockIdx.x; tile < total_tiles && alive; tile += gridDim.x) {
      const Tile t = decode<STAGE>(tile, tile_prefix, poff, row_off, g);
      if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u)) {
        report_error(g.err, kDevTimeoutMma);
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      for (int kb = 0; kb < t.nkb; ++kb) {
        if (!mbar_wait(&full_bar[stage], phase)) {
          report_error(g.err, kDevTimeoutMma);
          alive = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
        const uint32_t sb = sa + A_STAGE;
#pragma unroll
        for (int kk = 0; kk < BK / UK; ++kk) {
          const uint64_t ad = STAGE == kWgrad ? desc_mnmajor(sa + kk * UK * 128)
                                              : desc_kmajor(sa + kk * UK * 2);
          const uint64_t bd = (STAGE == kPre || STAGE == kWgrad) ? desc_mnmajor(sb + kk * UK * 128)
                                                                 : desc_kmajor(sb + kk * UK * 2);
          umma_bf16_ss(d_tmem, ad, bd, Idesc<STAGE>::value, (kb | kk) != 0 ? 1u : 0u);
        }
        umma_commit(&empty_bar[stage]);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!alive) break;
      umma_commit(&tfull_bar[acc]);   // with no k block (an expert without rows) it arrives at once
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    umma_commit(drain_bar);
    if (!mbar_wait(drain_bar, 0)) report_error(g.err, kDevTimeoutDrain);
  } else if (warp >= 2) {
    // ------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const Tile t = decode<STAGE>(tile, tile_prefix, poff, row_off, g);
      if (!mbar_wait(&tfull_bar[acc], acc_phase)) {
        report_error(g.err, kDevTimeoutEpilogue);
        break;
      }
      tc_fence_after_sync();
      const uint32_t tacc = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
      epilogue_tile<STAGE>(tacc, t, row, g);
      tc_fence_before_sync();
      mbar_arrive(&tempty_bar[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

bool encode2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_in,
              uint32_t box_out) {
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  const cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
  const cuuint32_t box[2] = {box_in, box_out};
  const cuuint32_t estr[2] = {1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// (E, rows, cols) bf16 row-major as a 3-D map {cols, rows, E}.
bool encode3d(CUtensorMap* m, const void* ptr, int E, uint64_t rows, uint64_t cols, uint32_t box_c,
              uint32_t box_r) {
  const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)E};
  const cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)rows * cols * 2};
  const cuuint32_t box[3] = {box_c, box_r, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int STAGE>
cudaError_t run_stage(const CUtensorMap& a, const CUtensorMap& a1, const CUtensorMap& b0,
                      const CUtensorMap& b1, const BwdArgs& g, int grid, cudaStream_t s) {
  auto kern = bwd_gemm_kernel<STAGE>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, grid, NUM_THREADS, SMEM_BYTES, s, 0, a, a1, b0, b1, g);
}

}  // namespace

int expert_backward_pad_rows(int rows_max, int E) {
  return rows_max + E * (kBwdPadRows - 1);
}

cudaError_t launch_expert_backward_gemms(const moe_config_t& c, const int32_t* offsets,
                                         const __nv_bfloat16* xp, const __nv_bfloat16* dyp,
                                         const __nv_bfloat16* W_in, const __nv_bfloat16* W_up,
                                         const __nv_bfloat16* W_out, float* pre,
                                         __nv_bfloat16* dab, __nv_bfloat16* hid, float* dx_perm,
                                         float* dW_in, float* dW_up, float* dW_out, int32_t* err,
                                         cudaStream_t s) {
  if (tensor_map_encoder() == nullptr) return cudaErrorNotSupported;
  const int E = c.E, d = c.d, DH = c.d_hidden, d_out = c.d_out;
  const int swiglu = c.expert_kind == MOE_EXPERT_SWIGLU ? 1 : 0;
  const int DHp = ceil_div(DH, 64) * 64;
  const int Rp = expert_backward_pad_rows(c.T * c.top_k, E);
  const int wide = (1 + swiglu) * DHp;   // columns of pre and dab
  BwdArgs g{};
  g.offsets = offsets;
  g.err = err;
  g.E = E;
  g.swiglu = swiglu;
  g.d = d;
  g.DH = DH;
  g.DHp = DHp;
  g.d_out = d_out;
  g.rows_max = c.T * c.top_k;
  g.pre = pre;
  g.dab = dab;
  g.hid = hid;
  g.dx = dx_perm;
  g.dw0 = dW_out;
  g.dw1 = dW_in;
  g.dw2 = dW_up;
  const int sms = device_sm_count();
  const int row_tiles_max = ceil_div(Rp, BM);
  CUtensorMap ta, ta1, tb0, tb1;
  cudaError_t e;

  // 1. pre = Xp [W_in | W_up]  (A K-major over Xp, B the weights as stored)
  if (c.T * c.top_k > 0) {
    g.K = d;
    g.N = DH;
    const int out_cols = swiglu ? BN / 2 : BN;
    g.n_tiles = ceil_div(DHp, out_cols);
    if (!encode2d(&ta, xp, d, Rp, BK, BM) || !encode3d(&tb0, W_in, E, d, DH, 64, BK) ||
        !encode3d(&tb1, swiglu ? W_up : W_in, E, d, DH, 64, BK))
      return cudaErrorInvalidValue;
    e = run_stage<kPre>(ta, ta, tb0, tb1, g,
                        (int)std::min<long>(sms, (long)(row_tiles_max + E) * g.n_tiles), s);
    if (e != cudaSuccess) return e;

    // 2. dH = dYp W_out^T; epilogue: dAB and H  (B K-major: W_out[e] rows)
    g.K = d_out;
    g.N = DH;
    g.n_tiles = ceil_div(DHp, BN);
    if (!encode2d(&ta, dyp, d_out, Rp, BK, BM) || !encode3d(&tb0, W_out, E, DH, d_out, BK, BN))
      return cudaErrorInvalidValue;
    e = run_stage<kDH>(ta, ta, tb0, tb0, g,
                       (int)std::min<long>(sms, (long)(row_tiles_max + E) * g.n_tiles), s);
    if (e != cudaSuccess) return e;

    // 3. dX = dAB [W_in | W_up]^T  (B K-major: W_in[e] / W_up[e] rows)
    g.K = wide;
    g.N = d;
    g.n_tiles = ceil_div(d, BN);
    if (!encode2d(&ta, dab, wide, Rp, BK, BM) || !encode3d(&tb0, W_in, E, d, DH, BK, BN) ||
        !encode3d(&tb1, swiglu ? W_up : W_in, E, d, DH, BK, BN))
      return cudaErrorInvalidValue;
    e = run_stage<kDX>(ta, ta, tb0, tb1, g,
                       (int)std::min<long>(sms, (long)(row_tiles_max + E) * g.n_tiles), s);
    if (e != cudaSuccess) return e;
  }

  // 4. dW_out = H^T dYp, dW_in = Xp^T dA, dW_up = Xp^T dB  (K = padded rows;
  //    an expert without rows gets a zero gradient)
  g.K = 0;
  g.N = 0;
  g.n_tiles = 0;
  const int rows_alloc = std::max(Rp, 1);
  if (!encode2d(&ta, hid, DHp, rows_alloc, 64, BK) || !encode2d(&ta1, xp, d, rows_alloc, 64, BK) ||
      !encode2d(&tb0, dyp, d_out, rows_alloc, 64, BK) ||
      !encode2d(&tb1, dab, wide, rows_alloc, 64, BK))
    return cudaErrorInvalidValue;
  long tiles = (long)E * ceil_div(DH, BM) * ceil_div(d_out, BN) +
               (long)(1 + swiglu) * E * ceil_div(d, BM) * ceil_div(DH, BN);
  return run_stage<kWgrad>(ta, ta1, tb0, tb1, g, (int)std::min<long>(sms, tiles), s);
}

}  // namespace moe
