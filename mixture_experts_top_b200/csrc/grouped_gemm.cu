// grouped_gemm.cu - ragged per-expert bf16 GEMM on Blackwell tensor cores
// (tcgen05 + tensor memory), with the expert activation fused into the
// epilogue.
//
// For every expert e the rows [offsets[e], offsets[e+1]) of A (the grouped
// token rows, K-major) are multiplied by that expert's weight matrix B_e
// (K, N), stored in the pages' x @ W orientation, i.e. N contiguous
// ("Mixture-of-Experts Routing - LLM Internals", mlgrind.dev, Algorithm 3 and
// Constraints: each expert runs only on its routed tokens).  Epilogues:
//   none   : out = acc, kept in fp32                    (down projection: the
//            expert output stays unrounded until the combine)
//   relu   : out = max(acc, 0)                          ("Mixture of Experts:
//            the Sparsely-Gated Layer", paperfordummies.in, The code,
//            `expert_forward`)
//   swiglu : out[:, c] = silu(acc_gate[:, c]) * acc_up[:, c]   (the SwiGLU
//            expert the pages name; silu(z) = z / (1 + exp(-z)))
//   scatter: the top-1 combine, gate * acc into the token's output row
//   combine: the top-k combine (Algorithm 3's gate-weighted sum): acc kept in
//            fp32 as for none, and the last of a token's kept rows to finish
//            an output column block sums the token's rows into its output
//
// B200 design
//  * One CTA per SM, persistent, 192 threads: warp 0 = TMA producer, warp 1 =
//    MMA issuer (one elected thread) and tensor-memory owner, warps 2-5 =
//    epilogue (each reads the 32 TMEM lanes its warp may access).
//  * Tile = 128 rows x 256 accumulator columns; k block 64; 4-stage smem ring
//    of 48 KiB stages (A 16 KiB + B 32 KiB), fed by TMA with 128-byte swizzle.
//    A is K-major; B is read straight from the (E, K, N) weights as an
//    N-major operand through a 3-D tensor map {N, K, E} (out-of-range K and N
//    are zero-filled, so ragged K and N tails need no special case).
//  * SwiGLU: the 256 accumulator columns are 128 gate columns followed by the
//    128 matching up columns (two 64-column boxes from each weight), so one
//    M128xN256xK16 instruction feeds both and the epilogue pairs them from
//    TMEM without any weight repacking.
//  * tcgen05.mma kind::f16 (bf16 in, fp32 accumulate) issued by one thread;
//    the accumulator lives in tensor memory, two buffers of 256 columns, so
//    the epilogue of one tile overlaps the main loop of the next.
//  * Tile order: expert-major, then output-column block, then row block, with
//    CTAs striding through it: CTAs running together share one weight column
//    block (read from HBM once, reused from L2) across the expert's row blocks.
//    Row tiles are re-read for every column block, so they are loaded with an
//    evict-last L2 policy; weights keep the normal policy (an evict-first
//    policy on them made CTAs that share a weight block re-read it from HBM,
//    and so did evict-first on only each block's last reader: 6.9 GB read
//    per Mixtral step against 5.4 GB).
//  * A tile that straddles two experts' rows reads the next expert's rows,
//    computes them, and masks them at the store: no padding of the grouped
//    layout is needed.
//  * Every mbarrier wait is bounded; on expiry the kernel records the error in
//    the workspace error word, drains its own copies and MMAs, frees tensor
//    memory and returns.
#include <cudaTypedefs.h>

#include <mutex>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int BM = 128;            // rows per tile (UMMA M)
constexpr int BK = 64;             // k per stage (one 128-byte swizzle row of bf16)
constexpr int BN = 256;            // accumulator columns per tile (UMMA N)
constexpr int UK = 16;             // k per tcgen05.mma (kind::f16)
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK * 2;          // 16 KiB
constexpr int B_BOX = 64 * BK * 2;            // one 64-column box: 8 KiB
constexpr int B_STAGE = BN * BK * 2;          // 32 KiB
constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 2 * BN;             // two accumulator buffers
constexpr int MAX_E = 256;
constexpr int AUX_BYTES = 4096;               // barriers, tmem address, tile table
// Row epilogues: per epilogue warp a 32 x 32 staging block (fp32 rows padded
// to 36 floats: conflict-free 16-byte writes by row and reads by column; bf16
// rows use it at 40 elements a row).
constexpr int EPI_LD = 36;
constexpr int EPI_BUF_BYTES = 4 * 32 * EPI_LD * 4;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + AUX_BYTES + EPI_BUF_BYTES;

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A bf16 (7-9 = 1),
// B bf16 (10-12 = 1), A K-major (bit 15 = 0), B N-major (bit 16 = 1),
// N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                            ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

// Shared-memory matrix descriptors (tcgen05): start address >> 4 at bits
// 0-13, leading byte offset >> 4 at 16-29, stride byte offset >> 4 at 32-45,
// version 1 at bit 46, swizzle mode at 61-63 (2 = 128-byte swizzle).
// A, K-major, 128B swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart
// (SBO); the leading offset is unused for this layout (set to 16 bytes).
__device__ __forceinline__ uint64_t desc_a_kmajor(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// B, N-major, 128B swizzle: each 64-column box is BK rows (k) of 128 bytes;
// 8-k-row groups are 1024 bytes apart (SBO); boxes along N are B_BOX bytes
// apart (LBO).
__device__ __forceinline__ uint64_t desc_b_nmajor(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(B_BOX >> 4) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

struct GemmArgs {
  const int32_t* offsets;
  const int32_t* perm;  // gathered A: grouped row r is row perm[r] of the A tensor (else null)
  int a_rows;           // rows of the A tensor (gathered A: tokens)
  void* out;  // bf16 for kEpiRelu / kEpiSwiglu / kEpiScatter / kEpiCombine, fp32 for kEpiNone
  int32_t* err;
  int E, K, N, rows_max;
  int n_tiles;  // output-column blocks
  // kEpiScatter / kEpiCombine (the combine in the epilogue): grouped row r
  // is a kept slot of token rows[r].  kEpiScatter (top_k = 1): the output
  // row is gates[token] * acc.  kEpiCombine: acc goes to row r of yrows, then
  // arrives on arrive[token * n_tiles + column block]; the last kept row of
  // the token to arrive writes the output block.
  const int32_t* rows;
  const float* gates;   // (T, top_k)
  const int32_t* dest;  // (T, top_k) grouped row of each slot, -1 if dropped
  int T, top_k;         // a token with no kept slot gets a zero output row
  float* yrows;
  unsigned* arrive;
  // Any kernel: clear_words words set to 0 before the first tile.
  unsigned* clear;
  size_t clear_words;
  // Pair kernel: [0] the next tile to hand out, [1] CTAs finished; both 0
  // at launch and left at 0 by the last CTA to finish.
  unsigned* sched;
  // Training forward (kEpiSwiglu / kEpiRelu, else null): every kept row's
  // fp32 pre-activations A (and B) are also written into the backward's
  // layout: blocks of kBwdPreBlock hidden units, block (p, u) = pre_Rp rows,
  // row = the row's padded row (each expert's rows rounded up to
  // kBwdPadRows, in expert order).
  float* pre;
  int pre_Rp, pre_mt;
};

// Padded row offsets of the backward's layout (each expert's rows rounded
// up to kBwdPadRows), by one warp: poff[e] for e = 0..E.
__device__ __forceinline__ void padded_offsets(const int* row_off, int E, bool ok, int lane,
                                               int* poff) {
  int carry = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    const int pr = (ok && e < E) ? (row_off[e + 1] - row_off[e] + kBwdPadRows - 1) / kBwdPadRows *
                                       kBwdPadRows
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
}

struct TileCoord {
  int e, m0, rows, n_tile;
};

template <int TILE_M = BM>
__device__ __forceinline__ TileCoord decode_tile(int tile, const int* prefix, const int* row_off,
                                                 int E, int n_tiles) {
  int lo = 0, hi = E;  // prefix[lo] <= tile < prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= tile) lo = mid; else hi = mid;
  }
  const int local = tile - prefix[lo];
  const int mt = (prefix[lo + 1] - prefix[lo]) / n_tiles;
  TileCoord c;
  c.e = lo;
  c.n_tile = local / mt;
  c.m0 = row_off[lo] + (local % mt) * TILE_M;
  c.rows = min(TILE_M, row_off[lo + 1] - c.m0);
  return c;
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }

// fp32 rows out of the epilogue, coalesced: the warp's 32 rows (lane = row,
// v32 = its columns [col, col + 32)) go through the warp's staging block and
// leave as 128-byte row segments, 8 lanes per row and 4 rows per store, rather
// than as 32 scattered 16-byte pieces per store.  roff[i] / rok[i]: element
// offset and validity of row 4 i + lane / 8 (from tile_row_slots).
// STREAM: evict-first stores (data read much later, e.g. by the backward).
// The segment of row i lands at base + roff[i] + col; col_n is its column in
// the matrix of N columns (the guard), equal to col except in blocked layouts.
template <bool STREAM = false>
__device__ __forceinline__ void store_rows_f32(float* wbuf, const uint32_t (&v32)[32], float* base,
                                               const size_t (&roff)[8], const bool (&rok)[8],
                                               int col, int N, int lane, int col_n = -1) {
  uint4* wrow = reinterpret_cast<uint4*>(wbuf + lane * EPI_LD);
#pragma unroll
  for (int v = 0; v < 8; ++v)
    wrow[v] = make_uint4(v32[4 * v], v32[4 * v + 1], v32[4 * v + 2], v32[4 * v + 3]);
  __syncwarp();
  const int c4 = lane & 7;
  const bool col_ok = (col_n < 0 ? col : col_n) + 4 * c4 < N;   // N is a multiple of 8
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint4 val = *reinterpret_cast<const uint4*>(wbuf + (4 * i + (lane >> 3)) * EPI_LD + 4 * c4);
    if (rok[i] && col_ok) {
      uint4* dst = reinterpret_cast<uint4*>(base + roff[i] + col + 4 * c4);
      if (STREAM)
        __stcs(dst, val);
      else
        *dst = val;
    }
  }
  __syncwarp();
}

// The warp's rows' pre-activations for hidden units [h0, h0 + 32) of matrix
// p (0: A, 1: B), from 32 fp32 accumulator columns, through the staging
// block: proff[i] = padded row * kBwdPreBlock of the lane's store rows.  Read
// only by the backward, much later: streamed past L2 (evict first).
__device__ __forceinline__ void store_pre32(float* wbuf, const GemmArgs& g, int p, int h0,
                                            const uint32_t (&r)[32], const size_t (&proff)[8],
                                            const bool (&prok)[8], int lane) {
  float* base = g.pre + (size_t)(p * g.pre_mt + h0 / kBwdPreBlock) * g.pre_Rp * kBwdPreBlock;
  store_rows_f32<true>(wbuf, r, base, proff, prok, h0 % kBwdPreBlock, g.N, lane, h0);
}

// bf16 rows out of the epilogue, the same way: the warp's 32 rows of 32
// columns (pk = this lane's row, packed in pairs) leave as 64-byte row
// segments, 4 lanes per row and 8 rows per store.  Rows of the staging block
// are 80 bytes apart (conflict-free 16-byte writes by row).  roff[i] /
// rok[i]: row 8 i + lane / 4, from tile_row_slots_bf16.
constexpr int EPI_LD16 = 40;   // bf16 elements per staging row
__device__ __forceinline__ void store_rows_bf16(float* wbuf, const uint32_t (&pk)[16],
                                                __nv_bfloat16* base, const size_t (&roff)[4],
                                                const bool (&rok)[4], int col, int N, int lane) {
  __nv_bfloat16* buf = reinterpret_cast<__nv_bfloat16*>(wbuf);
  uint4* wrow = reinterpret_cast<uint4*>(buf + lane * EPI_LD16);
#pragma unroll
  for (int v = 0; v < 4; ++v) wrow[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
  __syncwarp();
  const int c8 = lane & 3;
  const bool col_ok = col + 8 * c8 < N;   // N is a multiple of 8
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 val =
        *reinterpret_cast<const uint4*>(buf + (8 * i + (lane >> 2)) * EPI_LD16 + 8 * c8);
    if (rok[i] && col_ok) *reinterpret_cast<uint4*>(base + roff[i] + col + 8 * c8) = val;
  }
  __syncwarp();
}

// Offsets and validity of the rows this lane stores in store_rows_bf16: row
// 8 i + lane / 4 of the warp's 32.
__device__ __forceinline__ void tile_row_slots_bf16(size_t off, bool ok, int lane,
                                                    size_t (&roff)[4], bool (&rok)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int src = 8 * i + (lane >> 2);
    roff[i] = __shfl_sync(0xffffffffu, (unsigned long long)off, src);
    rok[i] = __shfl_sync(0xffffffffu, ok ? 1 : 0, src) != 0;
  }
}

// Offsets (elements) and validity of the rows this lane stores in
// store_rows_f32: row 4 i + lane / 8 of the warp's 32, whose own lanes hold
// `off` and `ok`.
__device__ __forceinline__ void tile_row_slots(size_t off, bool ok, int lane, size_t (&roff)[8],
                                               bool (&rok)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int src = 4 * i + (lane >> 3);
    roff[i] = __shfl_sync(0xffffffffu, (unsigned long long)off, src);
    rok[i] = __shfl_sync(0xffffffffu, ok ? 1 : 0, src) != 0;
  }
}

// kEpiCombine: what a row's arrival left for the combine of its token.
struct CombineRow {
  int tok;
  bool last;    // this row completed its token's kept slots for the block
  int dj[8];    // the token's slots' grouped rows (-1: dropped or beyond top_k)
  float gj[8];  // and gates
};

// Epilogue of one accumulator row held by this thread (TMEM lane = tile row):
// reads the 256 accumulator columns in chunks of 32 and writes the row's
// output columns [n0, n0 + OUT_COLS) of `out` (row offset orow_off), masked to
// N.  Every lane of the warp executes the tensor-memory loads (they are
// warp-collective) and the staged stores; only rows with `valid` are written.
template <int EPI>
__device__ __forceinline__ void store_tile_rows(uint32_t tacc, bool valid, size_t orow_off, int n0,
                                                const GemmArgs& g, int prow = -1,
                                                CombineRow* cr = nullptr, float* wbuf = nullptr) {
  constexpr int OUT_COLS = (EPI == kEpiSwiglu) ? BN / 2 : BN;
  if (EPI == kEpiScatter) {
    // orow_off is the grouped row; its token's output row gets gate * acc,
    // one rounding to bf16 (the combine's fp32 product, then its rounding).
    int tok = 0;
    float gate = 0.f;
    if (valid) {
      tok = g.rows[orow_off];
      valid = tok >= 0 && tok < g.T;
      if (valid) gate = g.gates[tok];
    }
    size_t roff[4];
    bool rok[4];
    tile_row_slots_bf16((size_t)tok * g.N, valid, threadIdx.x & 31, roff, rok);
#pragma unroll 1
    for (int cc = 0; cc < OUT_COLS; cc += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tacc + cc, r);
      tmem_ld_wait();
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        pk[i] = pack_bf16x2(gate * __uint_as_float(r[2 * i]), gate * __uint_as_float(r[2 * i + 1]));
      store_rows_bf16(wbuf, pk, static_cast<__nv_bfloat16*>(g.out), roff, rok, n0 + cc, g.N,
                      threadIdx.x & 31);
    }
  } else if (EPI == kEpiCombine) {
    // orow_off is the grouped row r.  Its fp32 row goes to yrows (the
    // combine's operand, and the backward's); the row then counts itself on
    // its token's counter for this column block with release order.  The
    // arrival that completes the token's kept slots (acquire order: every
    // other kept row's block is visible) is marked in *cr; combine_last_rows
    // sums those tokens once the accumulator is released.  The staged store
    // writes row r's block from other lanes of the warp; the warp barrier
    // that ends it orders those writes before this lane's releasing add.
    const int r = (int)orow_off;
    int tok = 0;
    if (valid) {
      tok = g.rows[r];
      if (tok < 0 || tok >= g.T) {
        report_error(g.err, kDevBadPerm);
        valid = false;
        tok = 0;
      }
    }
    size_t roff[8];
    bool rok[8];
    tile_row_slots((size_t)r * g.N, valid, threadIdx.x & 31, roff, rok);
#pragma unroll 1
    for (int cc = 0; cc < OUT_COLS; cc += 32) {
      uint32_t v32[32];
      tmem_ld_32x32b_x32(tacc + cc, v32);
      tmem_ld_wait();
      store_rows_f32(wbuf, v32, g.yrows, roff, rok, n0 + cc, g.N, threadIdx.x & 31);
    }
    cr->tok = tok;
    cr->last = false;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      cr->dj[j] = -1;
      cr->gj[j] = 0.f;
    }
    if (valid) {
      int kept = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < g.top_k) {
          int dd = g.dest[(size_t)tok * g.top_k + j];
          if (dd >= g.rows_max) {
            report_error(g.err, kDevBadPerm);
            dd = -1;
          }
          cr->dj[j] = dd;
          cr->gj[j] = g.gates[(size_t)tok * g.top_k + j];
          kept += dd >= 0 ? 1 : 0;
        }
      }
      const uint32_t old =
          atom_add_acq_rel_gpu(g.arrive + (size_t)tok * g.n_tiles + n0 / BN, 1u);
      cr->last = old + 1u == (uint32_t)kept;
    }
  } else if (EPI == kEpiSwiglu) {
    size_t roff[4];
    bool rok[4];
    tile_row_slots_bf16(orow_off, valid, threadIdx.x & 31, roff, rok);
    const bool save = g.pre != nullptr;   // uniform: the training forward
    size_t proff[8];
    bool prok[8];
    if (save)
      tile_row_slots((size_t)(prow < 0 ? 0 : prow) * kBwdPreBlock, valid && prow >= 0,
                     threadIdx.x & 31, proff, prok);
#pragma unroll 1
    for (int cc = 0; cc < OUT_COLS; cc += 32) {
      uint32_t gr[32], ur[32];
      tmem_ld_32x32b_x32(tacc + cc, gr);
      tmem_ld_32x32b_x32(tacc + OUT_COLS + cc, ur);
      tmem_ld_wait();
      if (save) {
        store_pre32(wbuf, g, 0, n0 + cc, gr, proff, prok, threadIdx.x & 31);
        store_pre32(wbuf, g, 1, n0 + cc, ur, proff, prok, threadIdx.x & 31);
      }
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float h0 = silu_f(__uint_as_float(gr[2 * i])) * __uint_as_float(ur[2 * i]);
        const float h1 = silu_f(__uint_as_float(gr[2 * i + 1])) * __uint_as_float(ur[2 * i + 1]);
        pk[i] = pack_bf16x2(h0, h1);
      }
      store_rows_bf16(wbuf, pk, static_cast<__nv_bfloat16*>(g.out), roff, rok, n0 + cc, g.N,
                      threadIdx.x & 31);
    }
  } else if (EPI == kEpiNone) {
    size_t roff[8];
    bool rok[8];
    tile_row_slots(orow_off, valid, threadIdx.x & 31, roff, rok);
#pragma unroll 1
    for (int cc = 0; cc < OUT_COLS; cc += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tacc + cc, r);
      tmem_ld_wait();
      store_rows_f32(wbuf, r, static_cast<float*>(g.out), roff, rok, n0 + cc, g.N,
                     threadIdx.x & 31);
    }
  } else {
    size_t roff[4];
    bool rok[4];
    tile_row_slots_bf16(orow_off, valid, threadIdx.x & 31, roff, rok);
    const bool save = g.pre != nullptr;   // uniform: the training forward
    size_t proff[8];
    bool prok[8];
    if (save)
      tile_row_slots((size_t)(prow < 0 ? 0 : prow) * kBwdPreBlock, valid && prow >= 0,
                     threadIdx.x & 31, proff, prok);
#pragma unroll 1
    for (int cc = 0; cc < OUT_COLS; cc += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tacc + cc, r);
      tmem_ld_wait();
      if (save) store_pre32(wbuf, g, 0, n0 + cc, r, proff, prok, threadIdx.x & 31);
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float v0 = fmaxf(__uint_as_float(r[2 * i]), 0.f);
        const float v1 = fmaxf(__uint_as_float(r[2 * i + 1]), 0.f);
        pk[i] = pack_bf16x2(v0, v1);
      }
      store_rows_bf16(wbuf, pk, static_cast<__nv_bfloat16*>(g.out), roff, rok, n0 + cc, g.N,
                      threadIdx.x & 31);
    }
  }
}

// kEpiCombine, after the accumulator is released: the warp writes the
// output block [n0, n0 + BN) of every token one of its lanes completed, two
// tokens per round.  Each lane owns 8 columns, so every slot row is read as
// one coalesced 1 KiB segment, all of a round's rows in flight at once; each
// element is the combine's fp32 chain over the slots in increasing j, then
// one rounding to bf16.  The rows were written by this warp's lanes (ordered
// by the warp barrier) or released by other rows' arrivals, which the lane
// that completed the token acquired.
__device__ __forceinline__ void combine_last_rows(const GemmArgs& g, const CombineRow& cr, int n0,
                                                  int lane) {
  uint32_t m = __ballot_sync(0xffffffffu, cr.last);
  if (m == 0u) return;
  __syncwarp();
  const int col = n0 + 8 * lane;
  const bool colok = col < g.N;  // N is a multiple of 8: all 8 columns or none
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out);
  while (m != 0u) {
    int src[2];
    src[0] = __ffs(m) - 1;
    m &= m - 1u;
    const bool two = m != 0u;
    src[1] = two ? __ffs(m) - 1 : src[0];
    if (two) m &= m - 1u;
    int tok[2], d[2][8];
    float gg[2][8];
    float4 ya[2][8], yb[2][8];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      tok[p] = __shfl_sync(0xffffffffu, cr.tok, src[p]);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        d[p][j] = __shfl_sync(0xffffffffu, cr.dj[j], src[p]);
        gg[p][j] = __shfl_sync(0xffffffffu, cr.gj[j], src[p]);
      }
    }
#pragma unroll
    for (int p = 0; p < 2; ++p) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        ya[p][j] = yb[p][j] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (colok && (p == 0 || two) && d[p][j] >= 0) {
          const float4* y = reinterpret_cast<const float4*>(g.yrows + (size_t)d[p][j] * g.N + col);
          ya[p][j] = __ldcg(y);
          yb[p][j] = __ldcg(y + 1);
        }
      }
    }
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      if (!colok || (p == 1 && !two)) continue;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (d[p][j] < 0) continue;
        acc[0] = fmaf(gg[p][j], ya[p][j].x, acc[0]);
        acc[1] = fmaf(gg[p][j], ya[p][j].y, acc[1]);
        acc[2] = fmaf(gg[p][j], ya[p][j].z, acc[2]);
        acc[3] = fmaf(gg[p][j], ya[p][j].w, acc[3]);
        acc[4] = fmaf(gg[p][j], yb[p][j].x, acc[4]);
        acc[5] = fmaf(gg[p][j], yb[p][j].y, acc[5]);
        acc[6] = fmaf(gg[p][j], yb[p][j].z, acc[6]);
        acc[7] = fmaf(gg[p][j], yb[p][j].w, acc[7]);
      }
      *reinterpret_cast<uint4*>(out + (size_t)tok[p] * g.N + col) =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                     pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    }
  }
}

// kEpiScatter / kEpiCombine: the output rows of tokens with every slot
// dropped are zero; the epilogue warps of every CTA write a strided share of
// them before their first tile (no grouped row maps to such a token, so no
// tile writes it).
__device__ __forceinline__ void zero_dropped_rows(const GemmArgs& g, int warp, int lane) {
  const int w = (int)blockIdx.x * 4 + (warp - 2), nw = (int)gridDim.x * 4;
  __nv_bfloat16* out = static_cast<__nv_bfloat16*>(g.out);
  for (int t = w; t < g.T; t += nw) {
    bool kept = false;
    for (int j = 0; j < g.top_k; ++j) kept = kept || g.dest[(size_t)t * g.top_k + j] >= 0;
    if (kept) continue;
    uint4* row = reinterpret_cast<uint4*>(out + (size_t)t * g.N);
    for (int v = lane; v < g.N / 8; v += 32) row[v] = make_uint4(0, 0, 0, 0);
  }
}

// g.clear: the epilogue warps of every CTA zero a strided share of the words
// before their first tile.
__device__ __forceinline__ void clear_words(const GemmArgs& g, int warp, int lane) {
  const size_t i0 = ((size_t)blockIdx.x * 4 + (size_t)(warp - 2)) * 32 + (size_t)lane;
  const size_t n = (size_t)gridDim.x * 128;
  for (size_t i = i0; i < g.clear_words; i += n) g.clear[i] = 0u;
}

template <int EPI, bool GATHER>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, const GemmArgs g) {
  pdl_wait_and_release();
  constexpr int OUT_COLS = (EPI == kEpiSwiglu) ? BN / 2 : BN;  // output columns per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* drain_bar = tempty_bar + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain_bar + 1);
  int* tile_prefix = reinterpret_cast<int*>(tmem_holder + 4);  // MAX_E + 1
  int* row_off = tile_prefix + (MAX_E + 1);                      // MAX_E + 1
  int* poff = row_off + (MAX_E + 1);                             // MAX_E + 1 (training forward)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = g.E;

  // ---- prologue: tile table (warp 0), tensor memory (warp 1), barriers.
  if (warp == 0) {
    for (int e = lane; e <= E; e += 32) row_off[e] = g.offsets[e];
    __syncwarp();
    bool ok = true;
    for (int e = lane; e < E; e += 32) ok = ok && (row_off[e] <= row_off[e + 1]);
    if (lane == 0) ok = ok && row_off[0] == 0 && row_off[E] <= g.rows_max;
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0 && blockIdx.x == 0) report_error(g.err, kDevBadOffsets);
    int carry = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int mt = (ok && e < E) ? (row_off[e + 1] - row_off[e] + BM - 1) / BM : 0;
      int incl = mt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      if (e < E) tile_prefix[e + 1] = (carry + incl) * g.n_tiles;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (g.pre != nullptr) padded_offsets(row_off, E, ok, lane, poff);
    if (lane == 0) {
      tile_prefix[0] = 0;
      tma_prefetch_map(&tmA);
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
  const int total_tiles = tile_prefix[E];
  const int num_kb = (g.K + BK - 1) / BK;

  if (warp == 0 && (GATHER || lane == 0)) {
    // ------------------------------------------------------ TMA producer
    // Lane 0 waits for a free stage and issues the B copies (and, without
    // GATHER, the A tile).  With GATHER every lane of warp 0 fetches 4 of the
    // tile's 128 rows by index (grouped row m -> A row perm[m]).
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, last_phase = 0;
    bool alive = true;
    const uint64_t pol_a = l2_policy_evict_last(), pol_b = l2_policy_evict_normal();
    for (int tile = blockIdx.x; tile < total_tiles && alive; tile += gridDim.x) {
      const TileCoord c = decode_tile(tile, tile_prefix, row_off, E, g.n_tiles);
      const int n0 = c.n_tile * OUT_COLS;
      int r4[4] = {0, 0, 0, 0};
      if (GATHER) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = c.m0 + 4 * lane + i;
          int r = m < row_off[E] ? g.perm[m] : 0;   // rows past the last expert: any valid row
          if (r < 0 || r >= g.a_rows) {
            report_error(g.err, kDevBadPerm);
            r = 0;
          }
          r4[i] = r;
        }
      }
      for (int kb = 0; kb < num_kb; ++kb) {
        uint8_t* sa = smem + stage * STAGE_BYTES;
        uint8_t* sb = sa + A_STAGE;
        const int k0 = kb * BK;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait(&empty_bar[stage], phase ^ 1u);
          if (!ok) {
            report_error(g.err, kDevTimeoutProducer);
          } else {
            mbar_arrive_expect_tx(&full_bar[stage], STAGE_BYTES);
            if (!GATHER) tma_load_2d_hint(sa, &tmA, &full_bar[stage], k0, c.m0, pol_a);
            if (EPI == kEpiSwiglu) {
              tma_load_3d_hint(sb, &tmB0, &full_bar[stage], n0, k0, c.e, pol_b);
              tma_load_3d_hint(sb + B_BOX, &tmB0, &full_bar[stage], n0 + 64, k0, c.e, pol_b);
              tma_load_3d_hint(sb + 2 * B_BOX, &tmB1, &full_bar[stage], n0, k0, c.e, pol_b);
              tma_load_3d_hint(sb + 3 * B_BOX, &tmB1, &full_bar[stage], n0 + 64, k0, c.e, pol_b);
            } else {
#pragma unroll
              for (int i = 0; i < 4; ++i)
                tma_load_3d_hint(sb + i * B_BOX, &tmB0, &full_bar[stage], n0 + 64 * i, k0, c.e,
                                 pol_b);
            }
            issued_mask |= 1u << stage;
            last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
          }
        }
        if (GATHER) {
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (ok)
            tma_gather4_hint(sa + lane * 4 * (BK * 2), &tmA, &full_bar[stage], k0, r4[0], r4[1],
                             r4[2], r4[3], pol_a);
        }
        if (!ok) {
          alive = false;
          break;
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // Drain: every copy issued must have landed before exit.
    if (lane == 0)
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
      if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u)) {
        report_error(g.err, kDevTimeoutMma);
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      for (int kb = 0; kb < num_kb; ++kb) {
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
          umma_bf16_ss(d_tmem, desc_a_kmajor(sa + kk * UK * 2), desc_b_nmajor(sb + kk * UK * 128),
                       kIdesc, (kb | kk) != 0 ? 1u : 0u);
        }
        umma_commit(&empty_bar[stage]);  // frees the stage once these MMAs finish
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!alive) break;
      umma_commit(&tfull_bar[acc]);  // accumulator ready for the epilogue
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    // Drain: all MMAs issued by this thread complete before TMEM is freed.
    umma_commit(drain_bar);
    if (!mbar_wait(drain_bar, 0)) report_error(g.err, kDevTimeoutDrain);
  } else if (warp >= 2) {
    // ------------------------------------------------------ epilogue
    if (EPI == kEpiScatter || EPI == kEpiCombine) zero_dropped_rows(g, warp, lane);
    if (g.clear != nullptr) clear_words(g, warp, lane);
    float* wbuf = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES + AUX_BYTES) +
                  (warp - 2) * 32 * EPI_LD;
    const int q = warp & 3;               // TMEM lane quarter of this warp
    const int row = q * 32 + lane;        // row inside the tile
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const TileCoord c = decode_tile(tile, tile_prefix, row_off, E, g.n_tiles);
      const int n0 = c.n_tile * OUT_COLS;
      if (!mbar_wait(&tfull_bar[acc], acc_phase)) {
        report_error(g.err, kDevTimeoutEpilogue);
        break;
      }
      tc_fence_after_sync();
      const uint32_t tacc = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
      const bool valid = row < c.rows;
      const size_t orow_off = (EPI == kEpiScatter || EPI == kEpiCombine)
                                  ? (size_t)(c.m0 + (valid ? row : 0))
                                  : (size_t)(c.m0 + (valid ? row : 0)) * g.N;
      const int prow = g.pre != nullptr ? poff[c.e] + (c.m0 - row_off[c.e]) + row : -1;
      CombineRow cr;
      store_tile_rows<EPI>(tacc, valid, orow_off, n0, g, prow, &cr, wbuf);
      tc_fence_before_sync();
      mbar_arrive_relaxed(&tempty_bar[acc]);   // the tile's stores need not drain first
      if (EPI == kEpiCombine) combine_last_rows(g, cr, n0, lane);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  // ---- teardown
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}


// ---------------------------------------------------------------------------
// CTA-pair variant (cta_group::2): a cluster of two CTAs computes a tile of
// 256 rows x 256 accumulator columns.  Each CTA stages its own 128 rows of A
// and one half of B (128 columns: the gate half and the up half for SwiGLU,
// or the two column halves otherwise) per 64-wide k block, 32 KiB per stage
// and 6 stages; the leader CTA's single MMA thread issues
// tcgen05.mma.cta_group::2 (M256 N256 K16), which reads both CTAs' shared
// memory and writes each CTA's 128 accumulator rows into its own tensor
// memory.  Per CTA this moves two thirds of the bytes of the single-CTA tile
// for the same FLOPs.  Both CTAs' copies count their bytes on the leader's
// full barrier; the leader's commits are multicast to both CTAs' empty and
// accumulator-full barriers; both CTAs' epilogue warps release an
// accumulator by arriving on the leader's barrier.  No load is multicast.
// Tiles are handed out dynamically, in order: the leader's producer claims
// the next tile index from a counter in global memory and publishes it to
// both CTAs through a small queue in shared memory (the peer's copy written
// through distributed shared memory); every role of both CTAs takes its
// tiles from that queue.  Pairs that run together therefore always work on
// neighbouring tiles, which share weight and row blocks in L2, however far
// apart their earlier tiles took them.
// ---------------------------------------------------------------------------

constexpr int PBM = 2 * BM;                       // rows per pair tile
constexpr int kTileQ = 4;                         // tile indices published ahead
// Readers of each published tile index: the leader's MMA thread, the peer's
// producer, and the four epilogue warps of each CTA.
constexpr int kTileQConsumers = 1 + 1 + 4 + 4;
constexpr int P_STAGES = 6;
constexpr int P_STAGE_BYTES = A_STAGE + B_STAGE / 2;  // 32 KiB
constexpr int P_SMEM_BYTES = P_STAGES * P_STAGE_BYTES + 1024 + AUX_BYTES + EPI_BUF_BYTES;
constexpr uint32_t kIdescPair = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                                ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(PBM >> 4) << 24);

template <int EPI, bool GATHER>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB0,
                             const __grid_constant__ CUtensorMap tmB1, const GemmArgs g) {
  pdl_wait_and_release();
  constexpr int OUT_COLS = (EPI == kEpiSwiglu) ? BN / 2 : BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + P_STAGES * P_STAGE_BYTES);
  uint64_t* empty_bar = full_bar + P_STAGES;
  uint64_t* tfull_bar = empty_bar + P_STAGES;
  uint64_t* tempty_bar = tfull_bar + 2;
  uint64_t* drain_bar = tempty_bar + 2;
  uint64_t* tq_full = drain_bar + 1;         // [kTileQ] a tile index was published
  uint64_t* tq_empty = tq_full + kTileQ;     // [kTileQ] (leader) every consumer has read it
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tq_empty + kTileQ);
  int* tile_q = reinterpret_cast<int*>(tmem_holder + 4);         // kTileQ
  int* tile_prefix = tile_q + kTileQ;                            // MAX_E + 1
  int* row_off = tile_prefix + (MAX_E + 1);                      // MAX_E + 1
  int* poff = row_off + (MAX_E + 1);                             // MAX_E + 1 (training forward)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = g.E;
  const uint32_t rank = cluster_cta_rank();   // 0 = leader, 1 = peer

  if (warp == 0) {
    for (int e = lane; e <= E; e += 32) row_off[e] = g.offsets[e];
    __syncwarp();
    bool ok = true;
    for (int e = lane; e < E; e += 32) ok = ok && (row_off[e] <= row_off[e + 1]);
    if (lane == 0) ok = ok && row_off[0] == 0 && row_off[E] <= g.rows_max;
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0 && blockIdx.x == 0) report_error(g.err, kDevBadOffsets);
    int carry = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int mt = (ok && e < E) ? (row_off[e + 1] - row_off[e] + PBM - 1) / PBM : 0;
      int incl = mt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      if (e < E) tile_prefix[e + 1] = (carry + incl) * g.n_tiles;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (g.pre != nullptr) padded_offsets(row_off, E, ok, lane, poff);
    if (lane == 0) {
      tile_prefix[0] = 0;
      tma_prefetch_map(&tmA);
      tma_prefetch_map(&tmB0);
      tma_prefetch_map(&tmB1);
    }
  } else if (warp == 1) {
    tmem_alloc_pair(tmem_holder, TMEM_COLS);
    tmem_relinquish_pair();
  } else if (warp == 2 && lane == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull_bar[b], 1);
      mbar_init(&tempty_bar[b], 8);  // one arrive per epilogue warp of both CTAs
    }
    mbar_init(drain_bar, 1);
    for (int q = 0; q < kTileQ; ++q) {
      mbar_init(&tq_full[q], 1);
      mbar_init(&tq_empty[q], kTileQConsumers);
    }
    fence_mbar_init();
  }
  tc_fence_before_sync();
  cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_holder;
  const int total_tiles = tile_prefix[E];
  const int num_kb = (g.K + BK - 1) / BK;

  if (warp == 0 && (GATHER || lane == 0)) {
    // ------------------------------------------------ TMA producer (both)
    // As in the single-CTA kernel: lane 0 waits and issues B (and A unless
    // GATHER); with GATHER each lane of warp 0 fetches 4 of this CTA's 128
    // rows by index.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, last_phase = 0;
    bool alive = true;
    const CUtensorMap* bmap = (EPI == kEpiSwiglu && rank == 1) ? &tmB1 : &tmB0;
    const uint64_t pol_a = l2_policy_evict_last(), pol_b = l2_policy_evict_normal();
    // Tiles are handed out in order: the leader claims the next index from
    // the global counter (one claim ahead, so its latency hides behind a
    // tile) and publishes it to both CTAs' queues; the peer reads it there.
    unsigned next = 0;
    if (rank == 0 && lane == 0) next = atomicAdd(&g.sched[0], 1u);
    for (int i = 0; alive; ++i) {
      const int slot = i & (kTileQ - 1);
      const uint32_t qpar = (uint32_t)(i / kTileQ) & 1u;
      int tile = total_tiles;
      if (lane == 0) {
        if (rank == 0) {
          if (!mbar_wait(&tq_empty[slot], qpar ^ 1u)) {
            report_error(g.err, kDevTimeoutProducer);
            alive = false;
          } else {
            tile = next < (unsigned)total_tiles ? (int)next : total_tiles;
            tile_q[slot] = tile;
            st_cluster_u32(cluster_smem_addr(&tile_q[slot], 1), (uint32_t)tile);
            mbar_arrive(&tq_full[slot]);
            mbar_arrive_cluster(cluster_smem_addr(&tq_full[slot], 1));
            if (tile < total_tiles) next = atomicAdd(&g.sched[0], 1u);
          }
        } else {
          if (!mbar_wait_cluster(&tq_full[slot], qpar)) {
            report_error(g.err, kDevTimeoutProducer);
            alive = false;
          } else {
            tile = tile_q[slot];
            mbar_arrive_cluster(cluster_smem_addr(&tq_empty[slot], 0));
          }
        }
      }
      if (GATHER) {
        tile = __shfl_sync(0xffffffffu, tile, 0);
        alive = __shfl_sync(0xffffffffu, alive, 0);
      }
      if (!alive || tile >= total_tiles) break;
      const TileCoord c = decode_tile<PBM>(tile, tile_prefix, row_off, E, g.n_tiles);
      const int n0 = c.n_tile * OUT_COLS;
      // this CTA's B half: gate / up for SwiGLU, else the column halves
      const int nb = (EPI == kEpiSwiglu) ? n0 : n0 + (int)rank * (BN / 2);
      const int my_m = c.m0 + (int)rank * BM;
      int r4[4] = {0, 0, 0, 0};
      if (GATHER) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int m = my_m + 4 * lane + u;
          int r = m < row_off[E] ? g.perm[m] : 0;   // rows past the last expert: any valid row
          if (r < 0 || r >= g.a_rows) {
            report_error(g.err, kDevBadPerm);
            r = 0;
          }
          r4[u] = r;
        }
      }
      for (int kb = 0; kb < num_kb; ++kb) {
        uint8_t* sa = smem + stage * P_STAGE_BYTES;
        uint8_t* sb = sa + A_STAGE;
        const int k0 = kb * BK;
        bool ok = true;
        if (lane == 0) {
          ok = mbar_wait(&empty_bar[stage], phase ^ 1u);
          if (!ok) {
            report_error(g.err, kDevTimeoutProducer);
          } else {
            if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * P_STAGE_BYTES);
            if (!GATHER) tma_load_2d_pair(sa, &tmA, &full_bar[stage], k0, my_m, pol_a);
            tma_load_3d_pair(sb, bmap, &full_bar[stage], nb, k0, c.e, pol_b);
            tma_load_3d_pair(sb + B_BOX, bmap, &full_bar[stage], nb + 64, k0, c.e, pol_b);
            issued_mask |= 1u << stage;
            last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
          }
        }
        if (GATHER) {
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (ok)
            tma_gather4_pair(sa + lane * 4 * (BK * 2), &tmA, &full_bar[stage], k0, r4[0], r4[1],
                             r4[2], r4[3], pol_a);
        }
        if (!ok) {
          alive = false;
          break;
        }
        if (++stage == P_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    // Drain: the leader's full barriers count both CTAs' copies.
    if (rank == 0 && lane == 0)
      for (int s = 0; s < P_STAGES; ++s)
        if ((issued_mask >> s) & 1u)
          if (!mbar_wait(&full_bar[s], (last_phase >> s) & 1u)) report_error(g.err, kDevTimeoutDrain);
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ------------------------------------------------ MMA issuer (leader)
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool alive = true;
    for (int i = 0; alive; ++i) {
      const int slot = i & (kTileQ - 1);
      if (!mbar_wait(&tq_full[slot], (uint32_t)(i / kTileQ) & 1u)) {
        report_error(g.err, kDevTimeoutMma);
        break;
      }
      const int tile = tile_q[slot];
      mbar_arrive(&tq_empty[slot]);
      if (tile >= total_tiles) break;
      if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u)) {
        report_error(g.err, kDevTimeoutMma);
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      for (int kb = 0; kb < num_kb; ++kb) {
        if (!mbar_wait(&full_bar[stage], phase)) {
          report_error(g.err, kDevTimeoutMma);
          alive = false;
          break;
        }
        tc_fence_after_sync();
        const uint32_t sa = smem_u32(smem + stage * P_STAGE_BYTES);
        const uint32_t sb = sa + A_STAGE;
#pragma unroll
        for (int kk = 0; kk < BK / UK; ++kk)
          umma_bf16_ss_pair(d_tmem, desc_a_kmajor(sa + kk * UK * 2),
                            desc_b_nmajor(sb + kk * UK * 128), kIdescPair,
                            (kb | kk) != 0 ? 1u : 0u);
        umma_commit_pair(&empty_bar[stage], 0x3);  // frees the stage in both CTAs
        if (++stage == P_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!alive) break;
      umma_commit_pair(&tfull_bar[acc], 0x3);  // accumulator ready in both CTAs
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    umma_commit_pair(drain_bar, 0x1);
    if (!mbar_wait(drain_bar, 0)) report_error(g.err, kDevTimeoutDrain);
  } else if (warp >= 2) {
    // ------------------------------------------------ epilogue (both)
    if (EPI == kEpiScatter || EPI == kEpiCombine) zero_dropped_rows(g, warp, lane);
    if (g.clear != nullptr) clear_words(g, warp, lane);
    float* wbuf = reinterpret_cast<float*>(smem + P_STAGES * P_STAGE_BYTES + AUX_BYTES) +
                  (warp - 2) * 32 * EPI_LD;
    const int q = warp & 3;
    const int row = (int)rank * BM + q * 32 + lane;  // row inside the pair tile
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int i = 0;; ++i) {
      const int slot = i & (kTileQ - 1);
      if (!mbar_wait_cluster(&tq_full[slot], (uint32_t)(i / kTileQ) & 1u)) {
        report_error(g.err, kDevTimeoutEpilogue);
        break;
      }
      const int tile = tile_q[slot];
      __syncwarp();
      // relaxed, so that it does not wait for the previous tile's stores; the
      // condition on `tile` keeps it behind the slot's read
      if (lane == 0 && tile >= 0) mbar_arrive_cluster_relaxed(cluster_smem_addr(&tq_empty[slot], 0));
      if (tile >= total_tiles) break;
      const TileCoord c = decode_tile<PBM>(tile, tile_prefix, row_off, E, g.n_tiles);
      const int n0 = c.n_tile * OUT_COLS;
      if (!mbar_wait(&tfull_bar[acc], acc_phase)) {
        report_error(g.err, kDevTimeoutEpilogue);
        break;
      }
      tc_fence_after_sync();
      const uint32_t tacc = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
      const bool valid = row < c.rows;
      const size_t orow_off = (EPI == kEpiScatter || EPI == kEpiCombine)
                                  ? (size_t)(c.m0 + (valid ? row : 0))
                                  : (size_t)(c.m0 + (valid ? row : 0)) * g.N;
      const int prow = g.pre != nullptr ? poff[c.e] + (c.m0 - row_off[c.e]) + row : -1;
      CombineRow cr;
      store_tile_rows<EPI>(tacc, valid, orow_off, n0, g, prow, &cr, wbuf);
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_leader_relaxed(&tempty_bar[acc]);   // stores need not drain
      if (EPI == kEpiCombine) combine_last_rows(g, cr, n0, lane);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  // ---- teardown: both CTAs done with tensor memory and shared memory
  tc_fence_before_sync();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
  // Every claim of this launch precedes its CTA's arrival here, so the last
  // CTA to arrive puts the counter back to 0 for the next launch.
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(&g.sched[1], 1u) == gridDim.x - 1u) {
      atomicExch(&g.sched[0], 0u);
      atomicExch(&g.sched[1], 0u);
    }
  }
}

// A: (rows, K) bf16 row-major, box 64 (k) x 128 (rows), 128B swizzle.
// Gathered A (box_rows = 1): the box is one row high, fetched four rows at a
// time by index.
bool encode_a(CUtensorMap* m, const void* ptr, int rows, int K, int box_rows = BM) {
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  const cuuint32_t box[2] = {BK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// B: (E, K, N) bf16 row-major as a 3-D map {N, K, E}, box 64 (n) x 64 (k) x 1.
bool encode_b(CUtensorMap* m, const void* ptr, int E, int K, int N) {
  const cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)K, (cuuint64_t)E};
  const cuuint64_t strides[2] = {(cuuint64_t)N * 2, (cuuint64_t)K * (cuuint64_t)N * 2};
  const cuuint32_t box[3] = {64, BK, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return tensor_map_encoder()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, bool GATHER>
cudaError_t run_gemm(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                     const GemmArgs& g, int grid, cudaStream_t s) {
  auto kern = grouped_gemm_kernel<EPI, GATHER>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, grid, NUM_THREADS, SMEM_BYTES, s, 0, a, b0, b1, g);
}

template <int EPI, bool GATHER>
cudaError_t run_gemm_pair(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                          const GemmArgs& g, int pairs, cudaStream_t s) {
  auto kern = grouped_gemm_pair_kernel<EPI, GATHER>;
  cudaError_t e = ensure_smem_limit(reinterpret_cast<const void*>(kern), P_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, 2 * pairs, NUM_THREADS, P_SMEM_BYTES, s, 2, a, b0, b1, g);
}

}  // namespace

size_t grouped_gemm_arrive_words(int T, int N) {
  return (size_t)std::max(T, 0) * (size_t)ceil_div(std::max(N, 1), BN);
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

cudaError_t launch_grouped_gemm(int epi, const __nv_bfloat16* A, int rows_max, int K,
                                const __nv_bfloat16* B0, const __nv_bfloat16* B1, int N, int E,
                                const int32_t* offsets, void* out, int32_t* err, unsigned* sched,
                                cudaStream_t s, const int32_t* perm, int a_rows,
                                const ScatterCombine* sc, float* pre, unsigned* clear,
                                size_t clear_words) {
  if (rows_max == 0) return cudaSuccess;
  if (pre != nullptr && epi != kEpiSwiglu && epi != kEpiRelu) return cudaErrorInvalidValue;
  if (tensor_map_encoder() == nullptr) return cudaErrorNotSupported;
  const bool gather = perm != nullptr;
  if (gather && (epi == kEpiNone || epi == kEpiScatter || a_rows <= 0)) return cudaErrorInvalidValue;
  const bool combine = epi == kEpiScatter || epi == kEpiCombine;
  if (combine != (sc != nullptr)) return cudaErrorInvalidValue;
  if (combine && (sc->top_k < 1 || sc->top_k > 8 || (epi == kEpiScatter && sc->top_k != 1) ||
                  (epi == kEpiCombine && (sc->y == nullptr || sc->arrive == nullptr))))
    return cudaErrorInvalidValue;
  if (gather && epi == kEpiCombine) return cudaErrorInvalidValue;
  if ((clear == nullptr) != (clear_words == 0)) return cudaErrorInvalidValue;
  CUtensorMap ta, tb0, tb1;
  const bool a_ok = gather ? encode_a(&ta, A, a_rows, K, 1) : encode_a(&ta, A, rows_max, K);
  if (!a_ok || !encode_b(&tb0, B0, E, K, N) ||
      !encode_b(&tb1, B1 != nullptr ? B1 : B0, E, K, N))
    return cudaErrorInvalidValue;
  const int out_cols = epi == kEpiSwiglu ? BN / 2 : BN;
  GemmArgs g;
  g.offsets = offsets;
  g.perm = perm;
  g.a_rows = gather ? a_rows : rows_max;
  g.out = out;
  g.err = err;
  g.E = E;
  g.K = K;
  g.N = N;
  g.rows_max = rows_max;
  g.n_tiles = ceil_div(N, out_cols);
  g.rows = sc != nullptr ? sc->rows : nullptr;
  g.gates = sc != nullptr ? sc->gates : nullptr;
  g.dest = sc != nullptr ? sc->dest : nullptr;
  g.T = sc != nullptr ? sc->T : 0;
  g.top_k = sc != nullptr ? sc->top_k : 0;
  g.yrows = sc != nullptr ? sc->y : nullptr;
  g.arrive = sc != nullptr ? sc->arrive : nullptr;
  g.clear = clear;
  g.clear_words = clear_words;
  g.sched = sched;
  g.pre = pre;
  g.pre_Rp = pre != nullptr ? expert_backward_pad_rows(rows_max, E) : 0;
  g.pre_mt = ceil_div(N, kBwdPreBlock);
  // Expert groups of 1024 rows or more on average: CTA pairs (M = 256 tiles,
  // a third less traffic per CTA); smaller groups: single CTAs (M = 128
  // tiles waste fewer rows at group edges).
  if (rows_max >= 1024 * E) {
    if (sched == nullptr) return cudaErrorInvalidValue;
    const long max_pairs = (long)(ceil_div(rows_max, PBM) + E) * g.n_tiles;
    const int pairs = (int)std::min<long>((long)(device_sm_count() / 2), max_pairs);
    if (gather)
      return epi == kEpiSwiglu ? run_gemm_pair<kEpiSwiglu, true>(ta, tb0, tb1, g, pairs, s)
                               : run_gemm_pair<kEpiRelu, true>(ta, tb0, tb1, g, pairs, s);
    switch (epi) {
      case kEpiSwiglu: return run_gemm_pair<kEpiSwiglu, false>(ta, tb0, tb1, g, pairs, s);
      case kEpiRelu: return run_gemm_pair<kEpiRelu, false>(ta, tb0, tb1, g, pairs, s);
      case kEpiScatter: return run_gemm_pair<kEpiScatter, false>(ta, tb0, tb1, g, pairs, s);
      case kEpiCombine: return run_gemm_pair<kEpiCombine, false>(ta, tb0, tb1, g, pairs, s);
      default: return run_gemm_pair<kEpiNone, false>(ta, tb0, tb1, g, pairs, s);
    }
  }
  const long max_tiles = (long)(ceil_div(rows_max, BM) + E) * g.n_tiles;
  const int grid = (int)std::min<long>((long)device_sm_count(), max_tiles);
  if (gather)
    return epi == kEpiSwiglu ? run_gemm<kEpiSwiglu, true>(ta, tb0, tb1, g, grid, s)
                             : run_gemm<kEpiRelu, true>(ta, tb0, tb1, g, grid, s);
  switch (epi) {
    case kEpiSwiglu: return run_gemm<kEpiSwiglu, false>(ta, tb0, tb1, g, grid, s);
    case kEpiRelu: return run_gemm<kEpiRelu, false>(ta, tb0, tb1, g, grid, s);
    case kEpiScatter: return run_gemm<kEpiScatter, false>(ta, tb0, tb1, g, grid, s);
    case kEpiCombine: return run_gemm<kEpiCombine, false>(ta, tb0, tb1, g, grid, s);
    default: return run_gemm<kEpiNone, false>(ta, tb0, tb1, g, grid, s);
  }
}

}  // namespace moe
