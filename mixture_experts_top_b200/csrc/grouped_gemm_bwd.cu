// grouped_gemm_bwd.cu - the experts' backward on Blackwell tensor cores
// (tcgen05 CTA pairs + tensor memory): four grouped bf16 GEMMs with fp32
// accumulation.
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
// [p_e, p_e+1), p_e = sum over e' < e of ceil(rows_e' / 64) * 64, its rows
// first and zero rows after them.  The zero rows add nothing to any product
// (their pre-activations, dH, dA, dB and H are zero too).
//
// Each GEMM puts a weight dimension on the MMA's M, 256 per CTA pair
// (cta_group::2; each CTA holds 128 of them in its tensor memory), and the
// other operand on N, so that the epilogue's lanes run along the weight
// dimension and every global access of a warp is one contiguous run:
//   kPre   M = hidden units of W_in, then of W_up; N = the expert's rows;
//          K = d.  pre^T = [W_in | W_up]^T Xp^T, stored fp32 in blocks of 256
//          hidden units (each block's rows one after another), the tiles dH
//          reads back
//   kDH    M = hidden units; N = rows; K = d_out.  dH^T = W_out dYp^T; the
//          epilogue reads the rows' pre-activations and writes dAB = [dA | dB]
//          and H (bf16)
//   kDX    M = d; N = rows; K = 2 hidden (dA then dB).  dX^T = [W_in | W_up]
//          dAB^T, written as fp32 rows of the unpadded grouped layout
//   kWgrad M = weight rows, N = weight columns (256), K = the expert's padded
//          rows.  dW_out = H^T dYp, dW_in = Xp^T dA, dW_up = Xp^T dB (fp32),
//          stored from shared memory by TMA in 32 x 32 boxes
// A row tile takes up to 256 of an expert's padded rows (N = 64 .. 256), so
// no tile straddles two experts.  Operand majors: the weights as K-major
// (kDH, kDX: W read along its rows) or M-major (kPre: W read along its
// columns); rows K-major; kWgrad's activations M- and N-major (K runs down
// their rows).  All staged by TMA with 128-byte swizzle; the tensor core
// reads either major from shared memory, so nothing is transposed in memory.
//
// B200 design as in grouped_gemm.cu's pair kernel: persistent, one CTA pair
// per two SMs, warp 0 TMA producer (each CTA loads its 128 weight rows and
// its half of the N operand), warp 1 of the leader issues the pair MMAs and
// owns tensor memory, warps 2-9 of both CTAs are the epilogue (two per
// tensor-memory lane quarter, each on half of the tile's columns; warps 2-5
// for kWgrad); 6 stages of
// 32 KiB (5 for kWgrad, whose epilogue stages its output in shared memory),
// two 256-column accumulators; every wait bounded (the error word records a
// timeout, copies and MMAs are drained and tensor memory is freed).
#include <cudaTypedefs.h>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int BM = 128;                        // weight rows per CTA
constexpr int PM = 2 * BM;                     // weight rows per pair tile (UMMA M)
static_assert(PM == kBwdPreBlock, "the stored pre-activations are blocked by the pair tile");
constexpr int BK = 64;
constexpr int BN = 256;                        // tile columns, at most (UMMA N)
constexpr int UK = 16;
constexpr int A_STAGE = BM * BK * 2;           // 16 KiB: this CTA's weight rows
constexpr int B_STAGE = (BN / 2) * BK * 2;     // 16 KiB: this CTA's half of N
constexpr int BOX64 = 64 * BK * 2;             // one 64 x 64 box: 8 KiB
constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
constexpr int TMEM_COLS = 2 * BN;
constexpr int MAX_E = 256;
constexpr int AUX_BYTES = 6144;                // barriers, tmem address, offsets, tile table
constexpr int OUT_BOX = 32 * 32 * 4;           // one 32 x 32 fp32 output box: 4 KiB
constexpr int OUT_BYTES = 4 * 2 * OUT_BOX;     // two per epilogue warp (kWgrad)

enum BwdStage { kPre = 0, kDH = 1, kDX = 2, kWgrad = 3 };

template <int STAGE>
struct Cfg {
  static constexpr int STAGES = STAGE == kWgrad ? 5 : 6;
  static constexpr int OUT = STAGE == kWgrad ? OUT_BYTES : 0;
  // Epilogue warps per CTA: the row stages use two per tensor-memory lane
  // quarter, each taking half of the tile's columns, so twice as many of
  // the epilogue's global accesses are in flight; kWgrad keeps four (its
  // output boxes take shared memory).
  static constexpr int EPI_WARPS = STAGE == kWgrad ? 4 : 8;
  static constexpr int THREADS = 64 + 32 * EPI_WARPS;
  static constexpr int SMEM = STAGES * STAGE_BYTES + OUT + 1024 + AUX_BYTES;
  // Instruction descriptor, kind::f16 (bf16 x bf16 -> fp32), M = 256: D fp32
  // (bit 4), A bf16 (7-9 = 1), B bf16 (10-12 = 1), A major at bit 15 and B
  // major at bit 16 (0 = K-major, 1 = MN-major), M >> 4 at 24; N >> 3 at 17
  // is added per tile.
  static constexpr uint32_t a_mn = (STAGE == kPre || STAGE == kWgrad) ? 1u : 0u;
  static constexpr uint32_t b_mn = STAGE == kWgrad ? 1u : 0u;
  static constexpr uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (a_mn << 15) |
                                    (b_mn << 16) | ((uint32_t)(PM >> 4) << 24);
  static_assert(SMEM <= 227 * 1024, "shared memory");
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
  int E, K;                 // K: the row stages' contraction length
  int swiglu;
  int d, DH, DHp, d_out;    // DHp: DH rounded up to 64
  int m_tiles;              // row stages: M tiles per weight matrix
  int rows_max;             // rows of the unpadded grouped buffers (T * top_k)
  int Rp;                   // rows of the padded layout
  float* pre;               // fp32 pre-activations A, B in blocks of 256 hidden units:
                            // block (p, mt) is (Rp, 256), p = 0 A, 1 B
  __nv_bfloat16* dab;       // (Rp, (1 + swiglu) DHp): [dA | dB]
  __nv_bfloat16* hid;       // (Rp, DHp): H
  float* dx;                // (R, d): unpadded grouped rows
};

// Weight-gradient problems of kWgrad: p = 0 dW_out (M DH, N d_out), p = 1
// dW_in (M d, N DH), p = 2 dW_up (M d, N DH; SwiGLU only).
__device__ __forceinline__ void wgrad_shape(const BwdArgs& g, int p, int& M, int& N) {
  M = p == 0 ? g.DH : g.d;
  N = p == 0 ? g.d_out : g.DH;
}

struct Tile {
  int e;      // expert
  int p;      // kPre: 0 = W_in, 1 = W_up; kWgrad: the problem
  int m0;     // first weight row of the pair tile (within its matrix)
  int n0;     // row stages: first padded row of the tile, relative to the expert; kWgrad: column
  int n;      // columns of the tile (row stages: 64 .. 256; kWgrad: 256)
  int kb0;    // first k block (kWgrad: the expert's first padded row / BK)
  int nkb;    // k blocks
};

__device__ __forceinline__ float sigmoid_f(float a) { return __fdividef(1.0f, 1.0f + __expf(-a)); }

// Tile order: row stages expert -> M tile -> N tile (an expert's rows, a few
// MB, stay in L2 while its weight tiles pass over them); kWgrad problem ->
// expert -> the weight dimension with more blocks -> the one with fewer.
template <int STAGE>
__device__ __forceinline__ Tile decode(int tile, const int* prefix, const int* poff,
                                       const BwdArgs& g) {
  Tile t{};
  if (STAGE != kWgrad) {
    int lo = 0, hi = g.E;  // prefix[lo] <= tile < prefix[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (prefix[mid] <= tile) lo = mid; else hi = mid;
    }
    const int prows = poff[lo + 1] - poff[lo];
    const int nt = (prows + BN - 1) / BN;
    const int local = tile - prefix[lo];
    const int mt = local / nt;
    t.e = lo;
    t.p = STAGE == kPre ? mt / g.m_tiles : 0;
    t.m0 = (STAGE == kPre ? mt % g.m_tiles : mt) * PM;
    t.n0 = (local % nt) * BN;
    t.n = min(BN, prows - t.n0);
    t.kb0 = 0;
    t.nkb = (g.K + BK - 1) / BK;
  } else {
    int p = 0, base = 0;
    for (; p < 3; ++p) {
      int M, N;
      wgrad_shape(g, p, M, N);
      const int cnt = g.E * ((M + PM - 1) / PM) * ((N + BN - 1) / BN);
      if (tile < base + cnt) break;
      base += cnt;
    }
    int M, N;
    wgrad_shape(g, p, M, N);
    const int mt = (M + PM - 1) / PM, nt = (N + BN - 1) / BN;
    const int local = tile - base;
    t.p = p;
    t.e = local / (mt * nt);
    const int rem = local % (mt * nt);
    // the dimension with fewer blocks runs innermost: the concurrent tiles
    // then share a few blocks of the other operand and all of this one's
    if (nt <= mt) {
      t.m0 = (rem / nt) * PM;
      t.n0 = (rem % nt) * BN;
    } else {
      t.m0 = (rem % mt) * PM;
      t.n0 = (rem / mt) * BN;
    }
    t.n = BN;
    t.kb0 = poff[t.e] / BK;
    t.nkb = (poff[t.e + 1] - poff[t.e]) / BK;
  }
  return t;
}

// Row-stage epilogues.  The thread owns weight row m = t.m0 + mrow of the
// tile (its tensor-memory lane) and walks the tile's columns, 32 rows of the
// expert at a time; at each of them the warp touches 32 consecutive weight
// indices of one row.
template <int STAGE>
__device__ __forceinline__ void epilogue_rows(uint32_t tacc, const Tile& t, int mrow, int c_begin,
                                              int c_end, const int* poff, const int* row_off,
                                              const BwdArgs& g) {
  const int m = t.m0 + mrow;
  const size_t wide = (size_t)(g.swiglu ? 2 : 1) * g.DHp;
  const int prow0 = poff[t.e] + t.n0;    // padded row of the tile's first column
#pragma unroll 1
  for (int c0 = c_begin; c0 < c_end; c0 += 32) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(tacc + (uint32_t)c0, r);
    tmem_ld_wait();
    if (STAGE == kPre) {
      // the tile's block: its 256 hidden units of every row, one 1 KB run per
      // row, so the pair's warps write (and dH's read) whole runs in order
      float* base = g.pre + ((size_t)(t.p * g.m_tiles + t.m0 / PM) * g.Rp + prow0 + c0) * PM + mrow;
#pragma unroll
      for (int j = 0; j < 32; ++j) __stcs(base + (size_t)j * PM, __uint_as_float(r[j]));
    } else if (STAGE == kDH) {
      if (m < g.DHp && m >= g.DH) {
        // hidden units past DH (the 64-wide padding): zero gradients and H,
        // whatever the pre-activation blocks hold there
        const size_t row = (size_t)(prow0 + c0);
        const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
#pragma unroll 4
        for (int j = 0; j < 32; ++j) {
          g.dab[(row + j) * wide + m] = z;
          if (g.swiglu) g.dab[(row + j) * wide + g.DHp + m] = z;
          g.hid[(row + j) * (size_t)g.DHp + m] = z;
        }
      } else if (m < g.DHp) {
        const size_t row = (size_t)(prow0 + c0);
        const float* pa = g.pre + ((size_t)(t.m0 / PM) * g.Rp + row) * PM + mrow;
        const float* pb = g.pre + ((size_t)(g.m_tiles + t.m0 / PM) * g.Rp + row) * PM + mrow;
        float av[32], bv[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          // each read once: streamed (evict first)
          av[j] = __ldcs(pa + (size_t)j * PM);
          bv[j] = g.swiglu ? __ldcs(pb + (size_t)j * PM) : 0.f;
        }
        __nv_bfloat16* da = g.dab + row * wide + m;
        __nv_bfloat16* hh = g.hid + row * (size_t)g.DHp + m;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float a = av[j], dh = __uint_as_float(r[j]);
          float dA, dB, H;
          if (g.swiglu) {
            const float b = bv[j];
            const float s = sigmoid_f(a);
            const float silu = a * s;
            dA = dh * b * (s * (1.0f + a * (1.0f - s)));
            dB = dh * silu;
            H = silu * b;
          } else {
            dA = a > 0.0f ? dh : 0.0f;
            dB = 0.0f;
            H = fmaxf(a, 0.0f);
          }
          __stcs(da + (size_t)j * wide, __float2bfloat16_rn(dA));
          if (g.swiglu) __stcs(da + (size_t)j * wide + g.DHp, __float2bfloat16_rn(dB));
          __stcs(hh + (size_t)j * g.DHp, __float2bfloat16_rn(H));
        }
      }
    } else {   // kDX: padded row -> the expert's unpadded grouped row (zero rows skipped)
      const int rows = row_off[t.e + 1] - row_off[t.e];
      if (m < g.d) {
        float* base = g.dx + (size_t)row_off[t.e] * g.d + m;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int local = t.n0 + c0 + j;
          if (local < rows) __stcs(base + (size_t)local * g.d, __uint_as_float(r[j]));
        }
      }
    }
  }
}

// kWgrad epilogue: the warp's 32 weight rows, 32 columns at a time, written
// into one of its two 32 x 32 boxes in shared memory (128-byte swizzle: the
// 16-byte piece j of row r at position j ^ (r mod 8)) and stored by TMA
// (columns or rows outside the gradient are not written).  An expert
// without rows gets zeros.
__device__ __forceinline__ void epilogue_wgrad(uint32_t tacc, const Tile& t, int rank, int q,
                                               int lane, uint8_t* stage_out, int& nbox,
                                               const CUtensorMap* out_map) {
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 32) {
    uint32_t r[32];
    if (t.nkb > 0) {
      tmem_ld_32x32b_x32(tacc + (uint32_t)c0, r);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) r[i] = 0u;
    }
    uint8_t* box = stage_out + (nbox & 1) * OUT_BOX;
    if (lane == 0 && nbox >= 2) bulk_wait_group_read<1>();   // the box's previous store has read it
    __syncwarp();
    uint8_t* rowp = box + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
          make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      // written once, never read here: evict first, so they do not push the
      // operands that the neighbouring tiles reuse out of L2
      tma_store_3d(out_map, box, t.n0 + c0, t.m0 + rank * BM + q * 32, t.e,
                   l2_policy_evict_first());
      bulk_commit_group();
    }
    ++nbox;
  }
}

// Tensor maps: A and A1 (kDX: W_up beside W_in; kWgrad: Xp beside H), B and
// B1 (kWgrad: [dA | dB] beside dYp), O0..O2 (kWgrad: dW_out, dW_in, dW_up).
template <int STAGE>
__global__ void __launch_bounds__(Cfg<STAGE>::THREADS, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB1,
                    const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
                    const __grid_constant__ CUtensorMap tmO2, const BwdArgs g) {
  using C = Cfg<STAGE>;
  constexpr int ST = C::STAGES;
  pdl_wait_and_release();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* out_stage = smem + ST * STAGE_BYTES;                  // kWgrad: 4 x 2 boxes
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(out_stage + C::OUT);
  uint64_t* empty_bar = full_bar + ST;
  uint64_t* tfull_bar = empty_bar + ST;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* drain_bar = tempty_bar + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain_bar + 1);
  int* tile_prefix = reinterpret_cast<int*>(tmem_holder + 4);   // MAX_E + 1
  int* poff = tile_prefix + (MAX_E + 1);                         // MAX_E + 1
  int* row_off = poff + (MAX_E + 1);                             // MAX_E + 1

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = g.E;
  const int rank = (int)cluster_cta_rank();   // 0 = leader, 1 = peer
  const int pair = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;

  if (warp == 0) {
    // Row offsets, padded offsets (rows per expert rounded up to 64) and,
    // for the row stages, the tile prefix (expert-major).
    for (int e = lane; e <= E; e += 32) row_off[e] = g.offsets[e];
    __syncwarp();
    bool ok = true;
    for (int e = lane; e < E; e += 32) ok = ok && (row_off[e] <= row_off[e + 1]);
    if (lane == 0) ok = ok && row_off[0] == 0 && row_off[E] <= g.rows_max;
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0 && blockIdx.x == 0) report_error(g.err, kDevBadOffsets);
    const int mt_all = STAGE == kPre ? (1 + g.swiglu) * g.m_tiles : g.m_tiles;
    int carry_rows = 0, carry_tiles = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int pr = (ok && e < E) ? (row_off[e + 1] - row_off[e] + kBwdPadRows - 1) /
                                         kBwdPadRows * kBwdPadRows
                                   : 0;
      const int tl = STAGE == kWgrad ? 0 : mt_all * ((pr + BN - 1) / BN);
      int incl = pr, incl_t = tl;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        const int nt = __shfl_up_sync(0xffffffffu, incl_t, o);
        if (lane >= o) {
          incl += n;
          incl_t += nt;
        }
      }
      if (e < E) {
        poff[e + 1] = carry_rows + incl;
        tile_prefix[e + 1] = carry_tiles + incl_t;
      }
      carry_rows += __shfl_sync(0xffffffffu, incl, 31);
      carry_tiles += __shfl_sync(0xffffffffu, incl_t, 31);
    }
    if (lane == 0) {
      poff[0] = 0;
      tile_prefix[0] = 0;
      tma_prefetch_map(&tmA);
      tma_prefetch_map(&tmA1);
      tma_prefetch_map(&tmB);
      tma_prefetch_map(&tmB1);
      if (STAGE == kWgrad) {
        tma_prefetch_map(&tmO0);
        tma_prefetch_map(&tmO1);
        tma_prefetch_map(&tmO2);
      }
    }
  } else if (warp == 1) {
    tmem_alloc_pair(tmem_holder, TMEM_COLS);
    tmem_relinquish_pair();
  } else if (warp == 2 && lane == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 2 * C::EPI_WARPS);  // one arrive per epilogue warp of both CTAs
    }
    mbar_init(drain_bar, 1);
    fence_mbar_init();
  }
  tc_fence_before_sync();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;
  int total_tiles;
  if (STAGE == kWgrad) {
    total_tiles = 0;
    for (int p = 0; p < (g.swiglu ? 3 : 2); ++p) {
      int M, N;
      wgrad_shape(g, p, M, N);
      total_tiles += E * ((M + PM - 1) / PM) * ((N + BN - 1) / BN);
    }
  } else {
    total_tiles = tile_prefix[E];
  }

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------ TMA producer (both)
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, last_phase = 0;
    bool alive = true;
    const uint64_t keep = l2_policy_evict_last(), stream = l2_policy_evict_normal();
    for (int tile = pair; tile < total_tiles && alive; tile += npairs) {
      const Tile t = decode<STAGE>(tile, tile_prefix, poff, g);
      const int am = t.m0 + rank * BM;                 // this CTA's first weight row
      const int brow = poff[t.e] + t.n0 + rank * (t.n / 2);   // row stages: its first B row
      for (int kb = 0; kb < t.nkb; ++kb) {
        uint8_t* sa = smem + stage * STAGE_BYTES;
        uint8_t* sb = sa + A_STAGE;
        if (!mbar_wait(&empty_bar[stage], phase ^ 1u)) {
          report_error(g.err, kDevTimeoutProducer);
          alive = false;
          break;
        }
        if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * STAGE_BYTES);
        const int k0 = (t.kb0 + kb) * BK;
        if (STAGE == kPre) {
          // A: W_in / W_up columns am .. am + 127 (M-major), two 64-wide boxes
          const CUtensorMap* wm = t.p == 0 ? &tmA : &tmA1;
          tma_load_3d_pair(sa, wm, &full_bar[stage], am, k0, t.e, stream);
          tma_load_3d_pair(sa + BOX64, wm, &full_bar[stage], am + 64, k0, t.e, stream);
          tma_load_2d_pair(sb, &tmB, &full_bar[stage], k0, brow, keep);
        } else if (STAGE == kDH) {
          tma_load_3d_pair(sa, &tmA, &full_bar[stage], k0, am, t.e, stream);   // W_out rows
          tma_load_2d_pair(sb, &tmB, &full_bar[stage], k0, brow, keep);
        } else if (STAGE == kDX) {
          if (k0 < g.DHp)
            tma_load_3d_pair(sa, &tmA, &full_bar[stage], k0, am, t.e, stream);          // W_in rows
          else
            tma_load_3d_pair(sa, &tmA1, &full_bar[stage], k0 - g.DHp, am, t.e, stream); // W_up rows
          tma_load_2d_pair(sb, &tmB, &full_bar[stage], k0, brow, keep);
        } else {
          // A (M-major): H (p = 0) or Xp (p >= 1); B (N-major): dYp (p = 0)
          // or [dA | dB] columns (dA: p = 1, dB: p = 2); two 64-wide boxes each
          const CUtensorMap* amap = t.p == 0 ? &tmA : &tmA1;
          const CUtensorMap* bmap = t.p == 0 ? &tmB : &tmB1;
          const int bcol = (t.p == 2 ? g.DHp : 0) + t.n0 + rank * (BN / 2);
          tma_load_2d_pair(sa, amap, &full_bar[stage], am, k0, stream);
          tma_load_2d_pair(sa + BOX64, amap, &full_bar[stage], am + 64, k0, stream);
          tma_load_2d_pair(sb, bmap, &full_bar[stage], bcol, k0, stream);
          tma_load_2d_pair(sb + BOX64, bmap, &full_bar[stage], bcol + 64, k0, stream);
        }
        issued_mask |= 1u << stage;
        last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == ST) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // Drain: the leader's full barriers count both CTAs' copies.
    if (rank == 0)
      for (int s = 0; s < ST; ++s)
        if ((issued_mask >> s) & 1u)
          if (!mbar_wait(&full_bar[s], (last_phase >> s) & 1u)) report_error(g.err, kDevTimeoutDrain);
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------ MMA issuer (leader)
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool alive = true;
    for (int tile = pair; tile < total_tiles && alive; tile += npairs) {
      const Tile t = decode<STAGE>(tile, tile_prefix, poff, g);
      const uint32_t idesc = C::idesc | ((uint32_t)(t.n >> 3) << 17);
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
          const uint64_t ad = C::a_mn ? desc_mnmajor(sa + kk * UK * 128)
                                      : desc_kmajor(sa + kk * UK * 2);
          const uint64_t bd = C::b_mn ? desc_mnmajor(sb + kk * UK * 128)
                                      : desc_kmajor(sb + kk * UK * 2);
          umma_bf16_ss_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        umma_commit_pair(&empty_bar[stage], 0x3);  // frees the stage in both CTAs
        if (++stage == ST) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!alive) break;
      // with no k block (an expert without rows) it arrives at once
      umma_commit_pair(&tfull_bar[acc], 0x3);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    umma_commit_pair(drain_bar, 0x1);
    if (!mbar_wait(drain_bar, 0)) report_error(g.err, kDevTimeoutDrain);
  } else if (warp >= 2) {
    // ------------------------------------------------ epilogue (both)
    const int q = warp & 3;                       // tensor-memory lanes 32q .. 32q + 31
    const int half = (warp - 2) / 4;              // row stages: which half of the columns
    const int mrow = rank * BM + q * 32 + lane;   // weight row inside the pair tile
    uint8_t* my_out = out_stage + q * 2 * OUT_BOX;
    int nbox = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total_tiles; tile += npairs) {
      const Tile t = decode<STAGE>(tile, tile_prefix, poff, g);
      if (!mbar_wait(&tfull_bar[acc], acc_phase)) {
        report_error(g.err, kDevTimeoutEpilogue);
        break;
      }
      tc_fence_after_sync();
      const uint32_t tacc = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
      if (STAGE == kWgrad)
        epilogue_wgrad(tacc, t, rank, q, lane, my_out, nbox,
                       t.p == 0 ? &tmO0 : (t.p == 1 ? &tmO1 : &tmO2));
      else
        epilogue_rows<STAGE>(tacc, t, mrow, half * (t.n / 2), (half + 1) * (t.n / 2), poff,
                             row_off, g);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_leader_relaxed(&tempty_bar[acc]);   // stores need not drain
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (STAGE == kWgrad && lane == 0) bulk_wait_group_all();   // stores done before exit
  }

  // ---- teardown: both CTAs done with tensor memory and shared memory
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
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

// (E, rows, cols) fp32 row-major as a 3-D store map {cols, rows, E}, box
// 32 x 32, 128-byte swizzle (a box row is 128 bytes).
bool encode3d_out(CUtensorMap* m, float* ptr, int E, uint64_t rows, uint64_t cols) {
  const cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)E};
  const cuuint64_t strides[2] = {(cuuint64_t)cols * 4, (cuuint64_t)rows * cols * 4};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, ptr, dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_NONE,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int STAGE>
cudaError_t run_stage(const CUtensorMap& a, const CUtensorMap& a1, const CUtensorMap& b,
                      const CUtensorMap& b1, const CUtensorMap& o0, const CUtensorMap& o1,
                      const CUtensorMap& o2, const BwdArgs& g, long tiles, cudaStream_t s) {
  auto kern = bwd_gemm_kernel<STAGE>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), Cfg<STAGE>::SMEM);
  if (e != cudaSuccess) return e;
  const int pairs = (int)std::max(1L, std::min<long>(device_sm_count() / 2, tiles));
  return launch_kernel(kern, 2 * pairs, Cfg<STAGE>::THREADS, Cfg<STAGE>::SMEM, s, 2, a, a1, b, b1,
                       o0, o1, o2, g);
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
                                         cudaStream_t s, bool pre_saved) {
  if (tensor_map_encoder() == nullptr) return cudaErrorNotSupported;
  const int E = c.E, d = c.d, DH = c.d_hidden, d_out = c.d_out;
  const int swiglu = c.expert_kind == MOE_EXPERT_SWIGLU ? 1 : 0;
  const int DHp = ceil_div(DH, 64) * 64;
  const int Rp = expert_backward_pad_rows(c.T * c.top_k, E);
  const int rows_alloc = std::max(Rp, 1);
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
  g.Rp = Rp;
  g.pre = pre;
  g.dab = dab;
  g.hid = hid;
  g.dx = dx_perm;
  const long row_tiles_max = ceil_div(Rp, BN) + E;   // N tiles over all experts, at most
  CUtensorMap ta, ta1, tb, tb1, to0, to1, to2;
  cudaError_t e;

  if (c.T * c.top_k > 0 && !pre_saved) {
    // 1. pre^T = [W_in | W_up]^T Xp^T  (A M-major: the weights as stored; B: Xp rows)
    g.K = d;
    g.m_tiles = ceil_div(DH, PM);
    if (!encode3d(&ta, W_in, E, d, DH, 64, BK) ||
        !encode3d(&ta1, swiglu ? W_up : W_in, E, d, DH, 64, BK) ||
        !encode2d(&tb, xp, d, rows_alloc, BK, BN / 2))
      return cudaErrorInvalidValue;
    e = run_stage<kPre>(ta, ta1, tb, tb, ta, ta, ta, g, (1L + swiglu) * g.m_tiles * row_tiles_max,
                        s);
    if (e != cudaSuccess) return e;
  }
  if (c.T * c.top_k > 0) {

    // 2. dH^T = W_out dYp^T; epilogue: dAB and H  (A K-major: W_out[e] rows)
    g.K = d_out;
    g.m_tiles = ceil_div(DH, PM);
    if (!encode3d(&ta, W_out, E, DH, d_out, BK, BM) ||
        !encode2d(&tb, dyp, d_out, rows_alloc, BK, BN / 2))
      return cudaErrorInvalidValue;
    e = run_stage<kDH>(ta, ta, tb, tb, ta, ta, ta, g, (long)g.m_tiles * row_tiles_max, s);
    if (e != cudaSuccess) return e;

    // 3. dX^T = [W_in | W_up] dAB^T  (A K-major: W_in[e] / W_up[e] rows)
    g.K = wide;
    g.m_tiles = ceil_div(d, PM);
    if (!encode3d(&ta, W_in, E, d, DH, BK, BM) ||
        !encode3d(&ta1, swiglu ? W_up : W_in, E, d, DH, BK, BM) ||
        !encode2d(&tb, dab, wide, rows_alloc, BK, BN / 2))
      return cudaErrorInvalidValue;
    e = run_stage<kDX>(ta, ta1, tb, tb, ta, ta, ta, g, (long)g.m_tiles * row_tiles_max, s);
    if (e != cudaSuccess) return e;
  }

  // 4. dW_out = H^T dYp, dW_in = Xp^T dA, dW_up = Xp^T dB  (K = padded rows;
  //    an expert without rows gets a zero gradient)
  g.K = 0;
  g.m_tiles = 0;
  if (!encode2d(&ta, hid, DHp, rows_alloc, 64, BK) || !encode2d(&ta1, xp, d, rows_alloc, 64, BK) ||
      !encode2d(&tb, dyp, d_out, rows_alloc, 64, BK) ||
      !encode2d(&tb1, dab, wide, rows_alloc, 64, BK) ||
      !encode3d_out(&to0, dW_out, E, DH, d_out) || !encode3d_out(&to1, dW_in, E, d, DH) ||
      !encode3d_out(&to2, swiglu ? dW_up : dW_in, E, d, DH))
    return cudaErrorInvalidValue;
  const long tiles = (long)E * ceil_div(DH, PM) * ceil_div(d_out, BN) +
                     (long)(1 + swiglu) * E * ceil_div(d, PM) * ceil_div(DH, BN);
  return run_stage<kWgrad>(ta, ta1, tb, tb1, to0, to1, to2, g, tiles, s);
}

}  // namespace moe
