// fa_bwd_kernel.cuh - backward of the fused attention for sm_100a.
//
// The backward recomputes the attention weights from Q, K and the forward's
// per-row log-sum-exp instead of storing them (the recomputation the jsqmd.com
// page describes: memory stays O(N)). With P_ij = exp(scale q_i.k_j - LSE_i)
// over the visible keys, D_i = dO_i . O_i and dS = P (dP - D):
//   dV = P^T dO,   dP = dO V^T,   dQ = scale dS K,   dK = scale dS^T Q.
//
// Three kernels, no atomics (deterministic):
//   fa_bwd_prep_kernel   -D_i and -LSE_i log2(e) into a workspace padded to
//                        whole 128-row tiles (pad rows: D = 0, LSE = +inf, so
//                        their weights are exactly 0);
//   fa_bwd_dq_kernel     work items (128-query tile, b, h): S = Q K^T and
//                        dP = dO V^T into TMEM, dS = P (dP - D), dQ += dS K
//                        over the key tiles;
//   fa_bwd_dkdv_kernel   work items (128-key tile, b, K/V head): S^T = K Q^T
//                        and dP^T = V dO^T into TMEM, P^T and dS^T, dV += P^T dO
//                        and dK += dS^T Q over the query tiles of the group's
//                        query heads.
// The two gradient kernels are persistent: one CTA per SM works through the
// items (scheduling below), and each item's result depends only on the item,
// not on which CTA computed it.
//
// Both are warp-specialised: a TMA loader warp (the tile's two fixed operands
// once, the streamed ones through rings), an MMA warp (converged, one elected
// lane issues tcgen05.mma) and two compute warpgroups that split each
// 128-column score tile into halves (TMEM lane = row, warpgroup h = columns
// 64h .. 64h+63). A compute thread keeps its 64 weights P in registers
// between its two phases: A reads S and forms P, B reads dP and forms dS. The
// 16-bit MMA operands they produce go back to TMEM inside the half's own
// columns. Score products keep N = 128: the tensor cores read both operands
// of a shared-memory product from shared memory, and at N = 64 that read,
// not the math, sets the pace.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "fa_fwd_kernel.cuh"
#include "sm100.cuh"

namespace fa {
namespace bwd {

constexpr int kThreads = 320;  // warps 0-7: compute warpgroups 0 and 1, 8: MMA, 9: loader
constexpr int kMma = 8;        // warp index
constexpr int kLoad = 9;       // warp index
constexpr int kGroup = 16;     // heads per scheduling group (causal)
constexpr int kItemReaders = 9;  // warps that read each work-item slot: the MMA warp and the 8 compute warps

template <int D>
struct Cfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kSlabBytes = 128 * 128;
  static constexpr int kTileBytes = kHalves * kSlabBytes;
  // D = 64: TMEM holds two S^T buffers beside dP^T and the two 64-column
  // accumulators, so S^T(t+2) is issued as soon as dV(t) has read P^T(t); a
  // third ring stage keeps its operands loaded by then.
  static constexpr bool kDoubleS = D == 64;
  static constexpr int kSBufs = kDoubleS ? 2 : 1;
  static constexpr int kStages = kDoubleS ? 3 : 2;
  static constexpr int kXOff = 0;                              // fixed operands X1, X2
  static constexpr int kYOff = kXOff + 2 * kTileBytes;          // ring of (Y1, Y2) pairs
  static constexpr int kBarOff = kYOff + kStages * 2 * kTileBytes;
  static constexpr int kBarX = 0;
  static constexpr int kBarYFull = 1;                       // [kStages]
  static constexpr int kBarYEmpty = 1 + kStages;            // [kStages]
  static constexpr int kBarSFull = 1 + 2 * kStages;         // [kSBufs] scores S^T of buffer b in TMEM
  static constexpr int kBarDPFull = kBarSFull + kSBufs;     // dP^T in TMEM
  static constexpr int kBarA = kBarDPFull + 1;              // [kSBufs][2] phase A of warpgroup h on buffer b done (128 arrivals)
  static constexpr int kBarB = kBarA + 2 * kSBufs;          // [2] phase B of warpgroup h done (128 arrivals)
  static constexpr int kBarDone = kBarB + 2;                // last accumulating MMA of an item finished
  static constexpr int kBarDrain = kBarDone + 1;
  static constexpr int kBarXEmpty = kBarDrain + 1;          // last MMA reading X1, X2 of an item finished
  static constexpr int kBarAccEmpty = kBarXEmpty + 1;       // accumulators read out (256 arrivals)
  static constexpr int kBarItemFull = kBarAccEmpty + 1;     // [2] work-item slot written
  static constexpr int kBarItemEmpty = kBarItemFull + 2;    // [2] work-item slot read (kItemReaders arrivals)
  static constexpr int kNumBars = kBarItemEmpty + 2;
  static constexpr int kWsOff = kBarOff + 256;        // key side, per stage: -LSE log2(e) and -D of the 128 queries
  static constexpr int kWsBytes = 2 * 128 * 4;
  static constexpr int kMiscOff = kWsOff + kStages * kWsBytes;
  static_assert(kNumBars * 8 <= 256, "barrier area");
  static constexpr int kSmemBytes = kMiscOff + 32 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  // TMEM columns: S^T buffer b at col_s(b), dP^T, accumulators acc0 = dK, acc1 = dV.
  __host__ __device__ static constexpr uint32_t col_s(int b) { return 128u * static_cast<uint32_t>(b); }
  static constexpr uint32_t kColDP = 128 * kSBufs, kColAcc0 = kColDP + 128, kColAcc1 = kColAcc0 + D;
  static_assert(kColAcc1 + D <= 512, "TMEM budget");
};

// Shapes: q, o, dO, dQ [B, Nq, Hq, D]; k, v, dK, dV [B, Nk, Hkv, D] (dense), or
// packed sequences [total_q, Hq, D] and [total_k, Hkv, D] where sequence b
// owns query rows cu_q[b] .. cu_q[b+1]-1 and key rows cu_k[b] .. cu_k[b+1]-1.
// Query head h reads K/V head h / G (G = Hq / Hkv). Causal: key j is visible
// to query i iff j <= i + delta, delta = nk - nq (aligned at the bottom-right
// corner) for the sequence's lengths nq, nk.
struct Params {
  const int* cu_q;      // packed sequences: B+1 query row offsets (device memory); dense: null
  const int* cu_k;      // packed sequences: B+1 key row offsets
  int total_q, total_k; // rows of the query-side and key-side tensors
  const float* ws_d;    // [B*Hq, Npad]: -D_i = -dO_i . O_i (0 on pad rows)
  const float* ws_l;    // [B*Hq, Npad]: -LSE_i * log2(e) (-inf on pad rows and rows that see no key)
  uint16_t* out0;       // query side: dQ;   key side: dK
  uint16_t* out1;       // key side: dV
  int Nq, Nk;           // dense: the lengths; packed: upper bounds of every sequence's lengths
  int Hq, Hkv, G;
  int BH;               // heads of this kernel's grid: B * Hq (query side) or B * Hkv (key side)
  int Npad;             // Nq rounded up to whole 128-row tiles
  int n_tiles;          // tiles per head of this kernel's grid: query tiles (query side) or key tiles (key side)
  float scale_log2;     // scale * log2(e)
  float scale;
  int causal;
  unsigned long long wait_limit_ns;
  int n_items;          // work items of this kernel's grid: BH * n_tiles
  int* sched;           // work-item counter of this launch (zeroed before it)
  int wide_stores;      // out0 and out1 are 32-byte aligned: gradient rows leave in 32-byte stores
};

// One sequence's rows and lengths as a CTA sees them.
struct Seq {
  int q0, nq, k0, nk;  // query rows q0 .. q0+nq-1, key rows k0 .. k0+nk-1
  int n_qt, n_kt;      // their 128-row tiles
  int delta;           // nk - nq: causal offset
  bool ok;             // packed offsets consistent
};

__device__ __forceinline__ Seq resolve_seq(const Params& prm, int b) {
  Seq sq;
  if (prm.cu_q != nullptr) {
    sq.q0 = prm.cu_q[b];
    sq.nq = prm.cu_q[b + 1] - sq.q0;
    sq.k0 = prm.cu_k[b];
    sq.nk = prm.cu_k[b + 1] - sq.k0;
    sq.ok = sq.q0 >= 0 && sq.nq >= 0 && sq.nq <= prm.Nq && static_cast<int64_t>(sq.q0) + sq.nq <= prm.total_q &&
            sq.k0 >= 0 && sq.nk >= 0 && sq.nk <= prm.Nk && static_cast<int64_t>(sq.k0) + sq.nk <= prm.total_k;
  } else {
    sq.q0 = b * prm.Nq;
    sq.nq = prm.Nq;
    sq.k0 = b * prm.Nk;
    sq.nk = prm.Nk;
    sq.ok = true;
  }
  sq.n_qt = (sq.nq + kTile - 1) / kTile;
  sq.n_kt = (sq.nk + kTile - 1) / kTile;
  sq.delta = sq.nk - sq.nq;
  return sq;
}

// 64 bytes (32 16-bit values, packed in pairs) to global memory: two 32-byte
// stores when `wide` (dst 32-byte aligned), else four 16-byte ones. When the
// 32 lanes of a warp write 32 different rows, each store instruction costs
// the L1 one pass per row, so the wide form halves the passes.
__device__ __forceinline__ void store_row64(void* dst, const uint32_t (&pk)[16], bool wide) {
  if (wide) {
#pragma unroll
    for (int k = 0; k < 2; ++k)
      asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(static_cast<char*>(dst) + 32 * k),
                   "r"(pk[8 * k]), "r"(pk[8 * k + 1]), "r"(pk[8 * k + 2]), "r"(pk[8 * k + 3]), "r"(pk[8 * k + 4]),
                   "r"(pk[8 * k + 5]), "r"(pk[8 * k + 6]), "r"(pk[8 * k + 7])
                   : "memory");
  } else {
    uint4* d = static_cast<uint4*>(dst);
#pragma unroll
    for (int k = 0; k < 4; ++k) d[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
  }
}

// -D_i and -LSE_i log2(e) per row into the tile-padded workspace (negated:
// the kernels add them); pad rows get D = 0, LSE = +inf (weights exactly 0).
// Streaming work, bound by reading O and dO once: a grid of a few blocks per
// SM strides over items of kPrepRowsPerIter consecutive rows i of one (b, h);
// D / 8 threads read a row's 16-byte pieces (each row is D * 2 contiguous
// bytes of [B, N, H, D]) and every thread keeps kPrepUnroll rows' loads in
// flight. Consecutive i keep the LSE reads and the workspace writes contiguous.
constexpr int kPrepUnroll = 4;
template <int D>
__host__ __device__ constexpr int prep_rows_per_iter() {
  return 8 * (32 / (D / 8)) * kPrepUnroll;  // 8 warps, 32 / (D / 8) rows per warp, kPrepUnroll deep
}

template <int D, bool FP16>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const uint16_t* __restrict__ o,
                                                          const uint16_t* __restrict__ dout,
                                                          const float* __restrict__ lse, float* __restrict__ ws_d,
                                                          float* __restrict__ ws_l, int B, int N, int H, int Npad,
                                                          int* __restrict__ sched) {
  constexpr int kLanes = D / 8;                 // threads per row
  constexpr int kRowsPerWarp = 32 / kLanes;
  constexpr int kRows = prep_rows_per_iter<D>();
  if (blockIdx.x == 0 && threadIdx.x < 2) sched[threadIdx.x] = 0;  // the gradient kernels' work-item counters
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32, sub = lane % kLanes;
  const int chunks = (N + kRows - 1) / kRows;
  const int64_t n_items = static_cast<int64_t>(B) * H * chunks;
  for (int64_t item = blockIdx.x; item < n_items; item += gridDim.x) {
    const int64_t bh = item / chunks;
    const int c = static_cast<int>(item - bh * chunks);
    const int64_t b = bh / H;
    const int h = static_cast<int>(bh - b * H);
    const int i0 = c * kRows + warp * kRowsPerWarp * kPrepUnroll + lane / kLanes;
    uint4 x[kPrepUnroll], y[kPrepUnroll];
#pragma unroll
    for (int u = 0; u < kPrepUnroll; ++u) {
      const int i = i0 + u * kRowsPerWarp;
      x[u] = make_uint4(0u, 0u, 0u, 0u);
      y[u] = x[u];
      if (i < N) {
        const int64_t row = (b * N + i) * H + h;
        x[u] = __ldg(reinterpret_cast<const uint4*>(o + row * D) + sub);
        y[u] = __ldg(reinterpret_cast<const uint4*>(dout + row * D) + sub);
      }
    }
#pragma unroll
    for (int u = 0; u < kPrepUnroll; ++u) {
      const int i = i0 + u * kRowsPerWarp;
      const uint32_t xs[4] = {x[u].x, x[u].y, x[u].z, x[u].w}, ys[4] = {y[u].x, y[u].y, y[u].z, y[u].w};
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 a = unpack2<FP16>(xs[k]);
        const float2 cc = unpack2<FP16>(ys[k]);
        acc = fmaf(a.x, cc.x, fmaf(a.y, cc.y, acc));
      }
#pragma unroll
      for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (i < N && sub == 0) {
        ws_d[bh * Npad + i] = -acc;
        // a row that sees no key has LSE = -inf: its weights are 0, not exp(+inf)
        const float l = lse[bh * N + i];
        ws_l[bh * Npad + i] = l == -INFINITY ? -INFINITY : -l * 1.44269504088896340736f;
      }
    }
  }
  const int pad = Npad - N;
  if (pad > 0) {
    const int64_t n_pad = static_cast<int64_t>(B) * H * pad;
    for (int64_t p = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; p < n_pad;
         p += static_cast<int64_t>(gridDim.x) * 256) {
      const int64_t idx = (p / pad) * Npad + N + p % pad;
      ws_d[idx] = 0.f;
      ws_l[idx] = -INFINITY;
    }
  }
}

// The same for packed sequences: O, dO [total_q, H, D], LSE [H, total_q],
// the workspace [B*H, Npad] per (sequence, head). Row r belongs to the sequence
// b with cu_q[b] <= r < cu_q[b+1] (binary search over the offsets); blocks from
// n_real_blocks on fill each (sequence, head)'s pad rows nq .. Npad-1. With
// inconsistent offsets nothing outside the workspace is written (the main
// kernels report them).
template <int D, bool FP16>
__global__ void __launch_bounds__(256) fa_bwd_prep_varlen_kernel(const uint16_t* __restrict__ o,
                                                                 const uint16_t* __restrict__ dout,
                                                                 const float* __restrict__ lse,
                                                                 float* __restrict__ ws_d, float* __restrict__ ws_l,
                                                                 const int* __restrict__ cu_q, int B, int H,
                                                                 int total_q, int Npad, unsigned n_real_blocks,
                                                                 int* __restrict__ sched) {
  constexpr int kLanes = D / 8;
  constexpr int kRowsPerBlock = 256 / kLanes;
  if (blockIdx.x == 0 && threadIdx.x < 2) sched[threadIdx.x] = 0;  // the gradient kernels' work-item counters
  if (blockIdx.x < n_real_blocks) {
    const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock + threadIdx.x / kLanes;  // r H + h
    const int sub = threadIdx.x % kLanes;
    const bool valid = row < static_cast<int64_t>(total_q) * H;
    float acc = 0.f;
    if (valid) {
      const uint4 x = __ldg(reinterpret_cast<const uint4*>(o + row * D) + sub);
      const uint4 y = __ldg(reinterpret_cast<const uint4*>(dout + row * D) + sub);
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 a = unpack2<FP16>(xs[k]);
        const float2 c = unpack2<FP16>(ys[k]);
        acc = fmaf(a.x, c.x, fmaf(a.y, c.y, acc));
      }
    }
#pragma unroll
    for (int off = kLanes / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (valid && sub == 0) {
      const int h = static_cast<int>(row % H);
      const int r = static_cast<int>(row / H);
      int lo = 0, hi = B;  // last b with cu_q[b] <= r
      while (hi - lo > 1) {
        const int mid = (lo + hi) / 2;
        if (cu_q[mid] <= r) lo = mid; else hi = mid;
      }
      const int i = r - cu_q[lo];
      if (i >= 0 && i < Npad) {
        const int64_t at = (static_cast<int64_t>(lo) * H + h) * Npad + i;
        ws_d[at] = -acc;
        const float l = lse[static_cast<int64_t>(h) * total_q + r];
        ws_l[at] = l == -INFINITY ? -INFINITY : -l * 1.44269504088896340736f;
      }
    }
  } else {
    const int64_t p = static_cast<int64_t>(blockIdx.x - n_real_blocks) * 256 + threadIdx.x;
    if (p < static_cast<int64_t>(B) * H * Npad) {
      const int b = static_cast<int>(p / (static_cast<int64_t>(H) * Npad));
      const int i = static_cast<int>(p % Npad);
      const int nq = cu_q[b + 1] - cu_q[b];
      if (i >= nq || nq < 0) {
        ws_d[p] = 0.f;
        ws_l[p] = -INFINITY;
      }
    }
  }
}

// Phase A for one thread's half row: p = 2^(s c + nl) for the 64 scores of
// TMEM columns t_s .. t_s + 63 of the score buffer (two 32-column chunks). nl is -LSE log2(e):
// per row (query side, `nl_row`) or per column from shared memory (key side,
// `nl_col`). MASKED tiles (causal tiles the diagonal cuts, key j visible to
// query i iff j <= i + delta, or the ragged tail of the keys) zero the
// invisible entries through the exponent and use the MUFU exp only; other
// tiles send every second pair through the FMA-pipe polynomial (the
// backward's exp work per tile is MUFU-bound at one exp unit per SM
// sub-partition; half on the FMA pipe measured fastest of 25/37.5/50%). With PACK the
// 16-bit weights are stored to the half's first 32 columns (key side: P^T).
template <bool FP16, bool KV_SIDE, bool MASKED, bool PACK>
__device__ __forceinline__ void phase_a(uint32_t t_s, float c, float nl_row, const float* nl_col, int first_col,
                                        int row_abs, int n_valid, int causal, int delta, float (&p)[64]) {
  const float2 c2 = make_float2(c, c);
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    uint32_t sa[32];
    tmem_ld32(t_s + ch * 32, sa);
    tmem_wait_ld();
    uint32_t pk[16];
    float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int e = ch * 32 + 2 * q;  // element index in the half
      float2 nl;
      if constexpr (KV_SIDE) {  // 16-byte broadcast reads (the buffer is 16-byte aligned)
        if ((q & 1) == 0) v4 = *reinterpret_cast<const float4*>(nl_col + e);
        nl = (q & 1) ? make_float2(v4.z, v4.w) : make_float2(v4.x, v4.y);
      } else {
        nl = make_float2(nl_row, nl_row);
      }
      float2 x = ffma2(make_float2(__uint_as_float(sa[2 * q]), __uint_as_float(sa[2 * q + 1])), c2, nl);
      float2 pp;
      if constexpr (MASKED) {
        const int c0 = first_col + e;  // column index (query on the key side, key on the query side)
        bool v0, v1;
        if constexpr (KV_SIDE) {  // row = key row_abs, column = query c0; pad queries carry -inf through nl
          v0 = !causal || row_abs <= c0 + delta;
          v1 = !causal || row_abs <= c0 + 1 + delta;
        } else {                  // row = query row_abs, column = key c0 (n_valid keys)
          v0 = c0 < n_valid && (!causal || c0 <= row_abs + delta);
          v1 = c0 + 1 < n_valid && (!causal || c0 + 1 <= row_abs + delta);
        }
        x.x = v0 ? x.x : -INFINITY;
        x.y = v1 ? x.y : -INFINITY;
        pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
      } else {
        if ((q & 1) == 1) {
          pp = exp2_poly2(x);
        } else {
          pp = make_float2(ex2_approx(x.x), ex2_approx(x.y));
        }
      }
      p[e] = pp.x;
      p[e + 1] = pp.y;
      if constexpr (PACK) pk[q] = pack2<FP16>(pp.x, pp.y);
    }
    if constexpr (PACK) tmem_st16(t_s + ch * 16, pk);
  }
}

// Phase B for one thread's half row: ds = p (dp + nd) for the 64 dP values of
// TMEM columns t_dp .. (two chunks), nd = -D per row (query side) or per column
// (key side); the 16-bit dS pairs go to t_out .. t_out + 31.
template <bool FP16, bool KV_SIDE>
__device__ __forceinline__ void phase_b(uint32_t t_dp, uint32_t t_out, float nd_row, const float* nd_col,
                                        const float (&p)[64]) {
#pragma unroll
  for (int ch = 0; ch < 2; ++ch) {
    uint32_t sb[32];
    tmem_ld32(t_dp + ch * 32, sb);
    tmem_wait_ld();
    uint32_t pk[16];
    float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int e = ch * 32 + 2 * q;
      float2 nd;
      if constexpr (KV_SIDE) {
        if ((q & 1) == 0) v4 = *reinterpret_cast<const float4*>(nd_col + e);
        nd = (q & 1) ? make_float2(v4.z, v4.w) : make_float2(v4.x, v4.y);
      } else {
        nd = make_float2(nd_row, nd_row);
      }
      const float2 g = fadd2(make_float2(__uint_as_float(sb[2 * q]), __uint_as_float(sb[2 * q + 1])), nd);
      const float2 ds = fmul2(make_float2(p[e], p[e + 1]), g);
      pk[q] = pack2<FP16>(ds.x, ds.y);
    }
    tmem_st16(t_out + ch * 16, pk);
  }
}

// Persistent scheduling (both gradient kernels). A launch runs one CTA per SM
// (at most one per work item). A CTA's first item is its block index. With
// the causal mask every further one comes from the launch's counter (zeroed
// before the launch), so a CTA that finishes early takes the next item and
// the lightest items, last in the order, fill the tail; without it items cost
// the same and a CTA takes every gridDim-th. The loader warp draws the items and hands each
// to the MMA warp and the compute warps through a two-slot ring in shared
// memory (-1 once the items run out). The mbarrier phases run on across
// items, counted by running totals (tiles streamed, items with work), so the
// next item's fixed operands load and its first score products are issued
// while the compute warps still write out the current item's gradients.

// Loader warp: item x (or -1) into slot i % 2, once the readers are done with
// the item that slot held before.
__device__ __forceinline__ bool item_publish(volatile int* slots, uint32_t full0, uint32_t empty0, int i, int x,
                                             WaitCtl wc) {
  const int slot = i & 1;
  if (i >= 2 && !warp_wait_bar(empty0 + 8 * slot, static_cast<uint32_t>(((i >> 1) & 1) ^ 1), wc)) return false;
  if ((threadIdx.x & 31) == 0) {
    slots[slot] = x;
    mbar_arrive(full0 + 8 * slot);  // release: the slot's value is visible to the waiters
  }
  __syncwarp();
  return true;
}

// A reading warp: the item in slot i % 2 (-1: no more), or -2 if the CTA is aborting.
__device__ __forceinline__ int item_take(const volatile int* slots, uint32_t full0, uint32_t empty0, int i,
                                         WaitCtl wc) {
  const int slot = i & 1;
  if (!warp_wait_bar(full0 + 8 * slot, static_cast<uint32_t>((i >> 1) & 1), wc)) return -2;
  const int x = slots[slot];
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(empty0 + 8 * slot);
  return x;
}

// Loader warp: the CTA's next item after x. Non-causal items all cost the
// same: a fixed stride keeps the CTAs in step, so CTAs working on the same
// head ask for the same K/V (or Q/dO) tiles at about the same time and the
// L2 serves them together. Causal items differ in cost: the counter.
__device__ __forceinline__ int item_next(int* sched, int x, int causal) {
  if (!causal) return x + static_cast<int>(gridDim.x);
  int nx = 0;
  if ((threadIdx.x & 31) == 0) nx = static_cast<int>(gridDim.x) + atomicAdd(sched, 1);
  return __shfl_sync(0xffffffffu, nx, 0);
}

// Key side work item: a tile of 128 keys of one K/V head of one sequence.
// Causal work per tile is uneven (later key tiles are seen by fewer query
// tiles): items go in groups of kGroup heads, heaviest tiles first within a
// group, so the tail holds the short ones and a group's Q/dO stay
// L2-resident. Non-causal: head-major.
struct ItemKV {
  int tile, b, hk;
  Seq sq;
  int t_first, per_head;  // query tiles t_first .. n_qt-1 of each of the G query heads see some key of the tile
  int n_t;                // streamed (query head, query tile) pairs: G * per_head
  bool skip;              // no work: tile past the sequence's end, or inconsistent packed offsets
};

__device__ __forceinline__ ItemKV item_kv(const Params& prm, int x) {
  ItemKV it;
  int bh;
  if (prm.causal) {
    const int per_group = kGroup * prm.n_tiles;
    const int g = x / per_group;
    const int r = x % per_group;
    const int gsize = min(kGroup, prm.BH - g * kGroup);
    bh = g * kGroup + r % gsize;
    it.tile = r / gsize;
  } else {
    it.tile = x % prm.n_tiles;
    bh = x / prm.n_tiles;
  }
  it.b = bh / prm.Hkv;
  it.hk = bh % prm.Hkv;
  it.sq = resolve_seq(prm, it.b);
  it.skip = !it.sq.ok || it.tile >= it.sq.n_kt;
  // query tiles that see some key of this tile: from the one holding the first
  // query i with i + delta >= tile * 128 (causal) to the last
  it.t_first = 0;
  if (prm.causal) {
    const int i0 = it.tile * kTile - it.sq.delta;
    it.t_first = i0 <= 0 ? 0 : i0 / kTile;
  }
  it.per_head = it.skip ? 0 : max(0, it.sq.n_qt - it.t_first);
  it.n_t = prm.G * it.per_head;
  return it;
}

// Key side: items are tiles of 128 keys of one K/V head; X1 = K, X2 = V stay
// in shared memory for the item, and (Q_t, dO_t) stream through a two-stage
// ring, each stage with the tile's -LSE log2(e) and -D, as pairs u = (g, t):
// for each of the G query heads g that read this K/V head, the query tiles t
// whose queries see some key of the tile. dK and dV accumulate over all pairs
// in TMEM (a fixed order, no atomics); out0 = dK, out1 = dV.
// TMEM holds one S^T / dP^T pair beside the two accumulators, so the MMA warp
// interleaves consecutive tiles, S(0) dP(0) | dV(t) S(t+1) dK(t) dP(t+1) | ...,
// issuing each accumulating product per half as soon as that half is in TMEM.
template <int D, bool FP16>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_x1, const __grid_constant__ CUtensorMap tm_x2,
                       const __grid_constant__ CUtensorMap tm_y1, const __grid_constant__ CUtensorMap tm_y2,
                       const Params prm) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto x_smem = [&](int i) { return sbase + C::kXOff + i * C::kTileBytes; };
  auto y_smem = [&](int s, int i) { return sbase + C::kYOff + (2 * s + i) * C::kTileBytes; };
  auto bar = [&](int i) { return sbase + C::kBarOff + 8 * i; };
  auto ws_stage = [&](int s) { return sbase + C::kWsOff + s * C::kWsBytes; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  volatile int* item_slots = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 8);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int causal = prm.causal;

  if (threadIdx.x == 0) {
    mbar_init(bar(C::kBarX), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(C::kBarYFull + s), 1);
      mbar_init(bar(C::kBarYEmpty + s), 1);
    }
    for (int b = 0; b < C::kSBufs; ++b) {
      mbar_init(bar(C::kBarSFull + b), 1);
      for (int h = 0; h < 2; ++h) mbar_init(bar(C::kBarA + 2 * b + h), 128);
    }
    mbar_init(bar(C::kBarDPFull), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::kBarB + i), 128);
      mbar_init(bar(C::kBarItemFull + i), 1);
      mbar_init(bar(C::kBarItemEmpty + i), kItemReaders);
    }
    mbar_init(bar(C::kBarDone), 1);
    mbar_init(bar(C::kBarDrain), 1);
    mbar_init(bar(C::kBarXEmpty), 1);
    mbar_init(bar(C::kBarAccEmpty), 256);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kMma) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, prm.wait_limit_ns};
  const uint32_t full0 = bar(C::kBarItemFull), empty0 = bar(C::kBarItemEmpty);

  if (warp == kLoad) {
    // ------------------------------------------------------------ loader (converged warp)
    if (lane == 0) {
      tma_prefetch_desc(&tm_x1);
      tma_prefetch_desc(&tm_x2);
      tma_prefetch_desc(&tm_y1);
      tma_prefetch_desc(&tm_y2);
    }
    __syncwarp();
    int x = static_cast<int>(blockIdx.x);
    int yc = 0, xi = 0;  // (Q, dO) stages and (K, V) pairs loaded so far
    bool ok = true;
    for (int i = 0; ok; ++i) {
      ok = item_publish(item_slots, full0, empty0, i, x < prm.n_items ? x : -1, wc);
      if (!ok || x >= prm.n_items) break;
      const ItemKV it = item_kv(prm, x);
      if (it.n_t > 0) {
        // K, V of this item once the previous item's last score products have read theirs
        if (xi > 0 && !(ok = warp_wait_bar(bar(C::kBarXEmpty), static_cast<uint32_t>((xi - 1) & 1), wc))) break;
        const int krow = it.sq.k0 + it.tile * kTile;
        mbar_arrive_expect_tx_elect(bar(C::kBarX), 2 * C::kTileBytes);
        for (int hf = 0; hf < C::kHalves; ++hf) {
          tma_load_3d_elect(x_smem(0) + hf * C::kSlabBytes, &tm_x1, hf * 64, it.hk, krow, bar(C::kBarX));
          tma_load_3d_elect(x_smem(1) + hf * C::kSlabBytes, &tm_x2, hf * 64, it.hk, krow, bar(C::kBarX));
        }
        ++xi;
        for (int u = 0; u < it.n_t; ++u, ++yc) {
          const int s = yc % C::kStages;
          if (yc >= C::kStages &&
              !(ok = warp_wait_bar(bar(C::kBarYEmpty + s), static_cast<uint32_t>(((yc / C::kStages) & 1) ^ 1), wc)))
            break;
          const int hq = it.hk * prm.G + u / it.per_head, tq = it.t_first + u % it.per_head;
          const int row = it.sq.q0 + tq * kTile;
          mbar_arrive_expect_tx_elect(bar(C::kBarYFull + s), 2 * C::kTileBytes + C::kWsBytes);
          for (int hf = 0; hf < C::kHalves; ++hf) {
            tma_load_3d_elect(y_smem(s, 0) + hf * C::kSlabBytes, &tm_y1, hf * 64, hq, row, bar(C::kBarYFull + s));
            tma_load_3d_elect(y_smem(s, 1) + hf * C::kSlabBytes, &tm_y2, hf * 64, hq, row, bar(C::kBarYFull + s));
          }
          // this query tile's -LSE log2(e) and -D ride with Q_t and dO_t
          const int64_t ws_row = (static_cast<int64_t>(it.b) * prm.Hq + hq) * prm.Npad + tq * kTile;
          bulk_load_elect(ws_stage(s), prm.ws_l + ws_row, kTile * 4, bar(C::kBarYFull + s));
          bulk_load_elect(ws_stage(s) + kTile * 4, prm.ws_d + ws_row, kTile * 4, bar(C::kBarYFull + s));
        }
        if (!ok) break;
      }
      x = item_next(prm.sched, x, causal);
    }
    // let the copies this warp issued land before shared memory is released
    if (xi > 0) drain_wait(bar(C::kBarX), static_cast<uint32_t>((xi - 1) & 1));
    for (int s = 0; s < C::kStages && s < yc; ++s) {
      const int last = s + ((yc - 1 - s) / C::kStages) * C::kStages;
      drain_wait(bar(C::kBarYFull + s), static_cast<uint32_t>((last / C::kStages) & 1));
    }
  } else if (warp == kMma) {
    // ------------------------------------------------------------ MMA issue (converged warp)
    constexpr uint32_t idesc_score = instr_desc_f16(kTile, kTile, FP16, false);
    constexpr uint32_t idesc_acc = instr_desc_f16(kTile, D, FP16, true);
    constexpr uint64_t kTileStep = C::kTileBytes >> 4;
    const uint64_t x_desc0 = smem_desc_sw128(x_smem(0), 16, 1024);  // K-major views
    const uint64_t y_desc0 = smem_desc_sw128(y_smem(0, 0), 16, 1024);
    const uint64_t y_mn0 = smem_desc_sw128(y_smem(0, 0), C::kSlabBytes, 1024);  // MN-major view of the same tiles
    // score product into TMEM column `col`: X_i Y_i(stage s)^T, K = D in steps of 16
    auto issue_score = [&](int i, int s, uint32_t col) {
      const uint64_t a = x_desc0 + static_cast<uint64_t>(i) * kTileStep;
      const uint64_t bb = y_desc0 + static_cast<uint64_t>(2 * s + i) * kTileStep;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>(((kk / 4) * C::kSlabBytes + (kk % 4) * 32) >> 4);
        mma_ss_elect(tmem + col, a + off, bb + off, idesc_score, kk > 0 ? 1u : 0u);
      }
    };
    // accumulating product for half hf of the streamed tile's 128 rows:
    // acc += A(TMEM, 16-bit pairs from a_col) * Y_i(stage s) rows 64hf .. (MN-major B)
    auto issue_acc = [&](uint32_t acc_col, uint32_t a_col, int i, int s, int hf, bool first) {
      const uint64_t bb = y_mn0 + static_cast<uint64_t>(2 * s + i) * kTileStep;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int kk = 4 * hf + q;
        mma_ts_elect(tmem + acc_col, tmem + a_col + q * 8, bb + static_cast<uint64_t>(kk * (2048 >> 4)), idesc_acc,
                     (first && q == 0) ? 0u : 1u);
      }
    };
    int yc = 0, tc = 0, xi = 0;  // streamed stages, score tiles and items with work so far
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int x = item_take(item_slots, full0, empty0, i, wc);
      if (x < 0) {
        ok = x == -1;
        break;
      }
      const ItemKV it = item_kv(prm, x);
      const int n = it.n_t;
      if (n == 0) continue;
      auto ystage = [&](int t) { return (yc + t) % C::kStages; };
      auto yphase = [&](int t) { return static_cast<uint32_t>(((yc + t) / C::kStages) & 1); };
      ok = warp_wait_bar(bar(C::kBarX), static_cast<uint32_t>(xi & 1), wc) &&
           warp_wait_bar(bar(C::kBarYFull + ystage(0)), yphase(0), wc);
      if (!ok) break;
      // score tile T (counted across items) goes to S^T buffer T % kSBufs
      auto sbuf = [&](int t) { return (tc + t) % C::kSBufs; };
      auto issue_s = [&](int t) {
        issue_score(0, ystage(t), C::col_s(sbuf(t)));
        mma_commit_elect(bar(C::kBarSFull + sbuf(t)));
      };
      tc_fence_after();
      issue_s(0);
      issue_score(1, ystage(0), C::kColDP);
      mma_commit_elect(bar(C::kBarDPFull));
      if (n == 1) mma_commit_elect(bar(C::kBarXEmpty));  // K, V of this item: last readers issued
      if (C::kDoubleS && n > 1) {
        ok = warp_wait_bar(bar(C::kBarYFull + ystage(1)), yphase(1), wc);
        if (!ok) break;
        tc_fence_after();
        issue_s(1);
      }
      for (int t = 0; ok && t < n; ++t) {
        const uint32_t ph = static_cast<uint32_t>((tc + t) & 1);
        const uint32_t pa = static_cast<uint32_t>(((tc + t) / C::kSBufs) & 1);  // phase of this tile's buffer
        const bool more = t + 1 < n;
        // dV += P^T dO per half as each warpgroup publishes its P^T; the first
        // one of an item waits until the previous item's accumulators are read out
        for (int hf = 0; hf < 2 && ok; ++hf) {
          ok = warp_wait_bar(bar(C::kBarA + 2 * sbuf(t) + hf), pa, wc);
          if (ok && t == 0 && hf == 0 && xi > 0)
            ok = warp_wait_bar(bar(C::kBarAccEmpty), static_cast<uint32_t>((xi - 1) & 1), wc);
          if (ok) {
            tc_fence_after();
            issue_acc(C::kColAcc1, C::col_s(sbuf(t)) + 64 * hf, 1, ystage(t), hf, t == 0 && hf == 0);
          }
        }
        if (!ok) break;
        // one buffer: S^T of the next tile (its P^T columns are free once dV has read them: in-order)
        if (!C::kDoubleS && more) {
          ok = warp_wait_bar(bar(C::kBarYFull + ystage(t + 1)), yphase(t + 1), wc);
          if (!ok) break;
          tc_fence_after();
          issue_s(t + 1);
        }
        // dK += dS^T Q per half
        for (int hf = 0; hf < 2 && ok; ++hf) {
          ok = warp_wait_bar(bar(C::kBarB + hf), ph, wc);
          if (ok) {
            tc_fence_after();
            issue_acc(C::kColAcc0, C::kColDP + 64 * hf, 0, ystage(t), hf, t == 0 && hf == 0);
          }
        }
        if (!ok) break;
        mma_commit_elect(bar(C::kBarYEmpty + ystage(t)));  // stage t: last reader issued
        if (more) {
          // dP of the next tile (after the accumulating products that read this tile's dS)
          issue_score(1, ystage(t + 1), C::kColDP);
          mma_commit_elect(bar(C::kBarDPFull));
          if (t + 1 == n - 1) mma_commit_elect(bar(C::kBarXEmpty));
          // two buffers: S^T two tiles ahead, into the buffer whose P^T dV(t) has read (in order)
          if (C::kDoubleS && t + 2 < n) {
            ok = warp_wait_bar(bar(C::kBarYFull + ystage(t + 2)), yphase(t + 2), wc);
            if (!ok) break;
            tc_fence_after();
            issue_s(t + 2);
          }
        } else {
          mma_commit_elect(bar(C::kBarDone));
        }
      }
      yc += n;
      tc += n;
      ++xi;
    }
    if (!ok) {
      mma_commit_elect(bar(C::kBarDrain));
      drain_wait(bar(C::kBarDrain), 0);
    }
  } else {
    // ------------------------------------------------------------ compute warpgroups (TMEM lane = row)
    const int wg = warp / 4;                  // column half of every score tile
    const int qd = warp % 4;                  // TMEM lane quadrant
    const int row = qd * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
    const float c = prm.scale_log2;
    const float nl_row = 0.f, nd_row = 0.f;  // per-column values on this side
    const uint32_t t_dp = tmem + lane_base + C::kColDP + 64 * wg;
    const uint32_t t_ds = t_dp;  // dS^T pairs over the first half of this half of dP^T
    int yc = 0, tc = 0, xi = 0;
    bool ok = true;
    int x = item_take(item_slots, full0, empty0, 0, wc);
    for (int i = 0; x >= 0; ++i) {
      const ItemKV it = item_kv(prm, x);
      if (it.skip) {
        if (!it.sq.ok && threadIdx.x == 0) atomicOr(&g_status_word, 2u);  // inconsistent packed offsets
        x = item_take(item_slots, full0, empty0, i + 1, wc);
        continue;
      }
      const int r_abs = it.tile * kTile + row;  // this thread's key
      for (int t = 0; t < it.n_t; ++t) {
        const int g = yc + t;
        const int s = g % C::kStages;
        const uint32_t ph = static_cast<uint32_t>((tc + t) & 1);
        const int sb = (tc + t) % C::kSBufs;                                   // this tile's S^T buffer
        const uint32_t pa = static_cast<uint32_t>(((tc + t) / C::kSBufs) & 1);  // and that buffer's phase
        const uint32_t t_s = tmem + lane_base + C::col_s(sb) + 64 * wg;
        const int cbase = (it.t_first + t % it.per_head) * kTile;  // first query (column) of this pair's tile
        const int first_col = cbase + 64 * wg;
        // this tile's -LSE log2(e) and -D for the warpgroup's 64 query columns,
        // in the TMA stage (released after phase B)
        const float* nl_col = reinterpret_cast<const float*>(smem + C::kWsOff + s * C::kWsBytes) + 64 * wg;
        const float* nd_col = nl_col + kTile;
        // masked: the causal boundary cuts the tile (its last key is not seen by
        // its first query), or the queries run out
        const bool masked = (causal && it.tile * kTile + kTile - 1 > cbase + it.sq.delta) || cbase + kTile > it.sq.nq;
        ok = warp_wait_bar(bar(C::kBarYFull + s), static_cast<uint32_t>((g / C::kStages) & 1), wc);
        if (!ok) break;
        ok = warp_wait_bar(bar(C::kBarSFull + sb), pa, wc);
        if (!ok) break;
        tc_fence_after();
        float p[64];
        if (masked) {
          phase_a<FP16, true, true, true>(t_s, c, nl_row, nl_col, first_col, r_abs, it.sq.nq, causal, it.sq.delta, p);
        } else {
          phase_a<FP16, true, false, true>(t_s, c, nl_row, nl_col, first_col, r_abs, it.sq.nq, causal, it.sq.delta, p);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::kBarA + 2 * sb + wg));
        ok = warp_wait_bar(bar(C::kBarDPFull), ph, wc);
        if (!ok) break;
        tc_fence_after();
        phase_b<FP16, true>(t_dp, t_ds, nd_row, nd_col, p);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::kBarB + wg));
      }
      if (!ok) break;
      // the next item (published by now: this item's loads have all been issued)
      const int nx = item_take(item_slots, full0, empty0, i + 1, wc);
      if (it.n_t > 0 && !(ok = warp_wait_bar(bar(C::kBarDone), static_cast<uint32_t>(xi & 1), wc))) break;
      // warpgroup 0 writes dK (scaled), warpgroup 1 dV; no query sees these
      // keys when there were no pairs: both are 0. After the last read of the
      // accumulator it goes back to the MMA warp (the next item's first dV
      // waits for that and for this warpgroup's next phase A anyway).
      const bool row_valid =
          r_abs < it.sq.nk && index_ok(static_cast<int64_t>(it.sq.k0) + r_abs < prm.total_k && it.hk < prm.Hkv);
      uint16_t* dst_row =
          (wg == 1 ? prm.out1 : prm.out0) + ((static_cast<int64_t>(it.sq.k0) + r_abs) * prm.Hkv + it.hk) * D;
      const float mul = wg == 1 ? 1.f : prm.scale;
      const uint32_t acc = tmem + lane_base + (wg == 0 ? C::kColAcc0 : C::kColAcc1);
      if (it.n_t > 0) tc_fence_after();
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t pk[16];
        if (it.n_t > 0) {
          uint32_t a[32];
          tmem_ld32(acc + q * 32, a);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 16; ++k)
            pk[k] = pack2<FP16>(__uint_as_float(a[2 * k]) * mul, __uint_as_float(a[2 * k + 1]) * mul);
          if (q == D / 32 - 1) {
            tc_fence_before();
            mbar_arrive(bar(C::kBarAccEmpty));
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) pk[k] = 0u;
        }
        if (row_valid) store_row64(dst_row + q * 32, pk, prm.wide_stores != 0);
      }
      yc += it.n_t;
      tc += it.n_t;
      if (it.n_t > 0) ++xi;
      x = nx;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Query side work item: a tile of 128 queries of one query head of one
// sequence; causal in groups of kGroup heads with the heaviest (latest) tiles
// first, non-causal head-major.
struct ItemQ {
  int tile, bh, h, hk;
  Seq sq;
  int n_t;    // key tiles 0 .. n_t-1 (causal: up to the one holding the last key the tile's last query sees)
  bool skip;  // no work: tile past the sequence's end, or inconsistent packed offsets
};

__device__ __forceinline__ ItemQ item_q(const Params& prm, int x) {
  ItemQ it;
  if (prm.causal) {
    const int per_group = kGroup * prm.n_tiles;
    const int g = x / per_group;
    const int r = x % per_group;
    const int gsize = min(kGroup, prm.BH - g * kGroup);
    it.bh = g * kGroup + r % gsize;
    it.tile = prm.n_tiles - 1 - r / gsize;
  } else {
    it.tile = x % prm.n_tiles;
    it.bh = x / prm.n_tiles;
  }
  it.h = it.bh % prm.Hq;
  it.hk = it.h / prm.G;  // the K/V head this query head reads
  it.sq = resolve_seq(prm, it.bh / prm.Hq);
  it.skip = !it.sq.ok || it.tile >= it.sq.n_qt;
  it.n_t = it.skip ? 0 : it.sq.n_kt;
  if (!it.skip && prm.causal) {
    const int last_key = it.tile * kTile + kTile - 1 + it.sq.delta;
    it.n_t = last_key < 0 ? 0 : min(it.sq.n_kt, last_key / kTile + 1);
  }
  return it;
}

// Query side with a double-buffered score tile: items are tiles of 128
// queries of one query head; Q and dO stay in shared memory for the item, K_t
// streams through a three-stage ring and V_t through a two-stage ring. TMEM:
// S(t) in buffer t % 2 (columns 0 and 128; t counted across items), dP at 256,
// dQ at 384; dS(t) is written back over the first half of each warpgroup's
// columns of its own S buffer. The MMA warp waits once per streamed tile, for
// both warpgroups' dS(t), and then issues
//   dP(t+1), dQ(t), S(t+2)
// back to back, so the score product two tiles ahead is already in TMEM when
// the warpgroups need it.
template <int D>
struct CfgQ {
  static constexpr int kHalves = D / 64;
  static constexpr int kSlabBytes = 128 * 128;
  static constexpr int kTileBytes = kHalves * kSlabBytes;
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kXOff = 0;                                // Q, dO
  static constexpr int kKOff = kXOff + 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kVStages * kTileBytes;
  static constexpr int kBarX = 0;
  static constexpr int kBarKFull = 1;                             // [kKStages]
  static constexpr int kBarKEmpty = kBarKFull + kKStages;         // [kKStages]
  static constexpr int kBarVFull = kBarKEmpty + kKStages;         // [kVStages]
  static constexpr int kBarVEmpty = kBarVFull + kVStages;         // [kVStages]
  static constexpr int kBarSFull = kBarVEmpty + kVStages;         // [2] S buffer b holds S(t), t % 2 == b
  static constexpr int kBarDPFull = kBarSFull + 2;
  static constexpr int kBarB = kBarDPFull + 1;                    // [2] warpgroup h wrote dS(t) (128 arrivals)
  static constexpr int kBarDone = kBarB + 2;                      // last dQ product of an item finished
  static constexpr int kBarDrain = kBarDone + 1;
  static constexpr int kBarXEmpty = kBarDrain + 1;                // last MMA reading Q, dO of an item finished
  static constexpr int kBarAccEmpty = kBarXEmpty + 1;             // dQ accumulator read out (256 arrivals)
  static constexpr int kBarItemFull = kBarAccEmpty + 1;           // [2] work-item slot written
  static constexpr int kBarItemEmpty = kBarItemFull + 2;          // [2] work-item slot read (kItemReaders arrivals)
  static constexpr int kNumBars = kBarItemEmpty + 2;
  static_assert(kNumBars * 8 <= 256, "barrier area");
  static constexpr int kMiscOff = kBarOff + 256;
  static constexpr int kSmemBytes = kMiscOff + 32 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static constexpr uint32_t kColS0 = 0, kColDP = 256, kColAcc = 384;
  static_assert(384 + D <= 512, "TMEM budget");
};

template <int D, bool FP16>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const Params prm) {
  using C = CfgQ<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto x_smem = [&](int i) { return sbase + C::kXOff + i * C::kTileBytes; };
  auto k_smem = [&](int s) { return sbase + C::kKOff + s * C::kTileBytes; };
  auto v_smem = [&](int s) { return sbase + C::kVOff + s * C::kTileBytes; };
  auto bar = [&](int i) { return sbase + C::kBarOff + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  volatile int* item_slots = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 8);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int causal = prm.causal;

  if (threadIdx.x == 0) {
    mbar_init(bar(C::kBarX), 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(bar(C::kBarKFull + s), 1);
      mbar_init(bar(C::kBarKEmpty + s), 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(bar(C::kBarVFull + s), 1);
      mbar_init(bar(C::kBarVEmpty + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::kBarSFull + i), 1);
      mbar_init(bar(C::kBarB + i), 128);
      mbar_init(bar(C::kBarItemFull + i), 1);
      mbar_init(bar(C::kBarItemEmpty + i), kItemReaders);
    }
    mbar_init(bar(C::kBarDPFull), 1);
    mbar_init(bar(C::kBarDone), 1);
    mbar_init(bar(C::kBarDrain), 1);
    mbar_init(bar(C::kBarXEmpty), 1);
    mbar_init(bar(C::kBarAccEmpty), 256);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kMma) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, prm.wait_limit_ns};
  const uint32_t full0 = bar(C::kBarItemFull), empty0 = bar(C::kBarItemEmpty);

  if (warp == kLoad) {
    // ------------------------------------------------------------ loader (converged warp)
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
    }
    __syncwarp();
    int x = static_cast<int>(blockIdx.x);
    int kc = 0, vc = 0, xi = 0;  // K and V tiles and (Q, dO) pairs loaded so far
    bool ok = true;
    for (int i = 0; ok; ++i) {
      ok = item_publish(item_slots, full0, empty0, i, x < prm.n_items ? x : -1, wc);
      if (!ok || x >= prm.n_items) break;
      const ItemQ it = item_q(prm, x);
      if (it.n_t > 0) {
        // Q, dO of this item once the previous item's last products have read theirs
        if (xi > 0 && !(ok = warp_wait_bar(bar(C::kBarXEmpty), static_cast<uint32_t>((xi - 1) & 1), wc))) break;
        const int qrow = it.sq.q0 + it.tile * kTile;
        mbar_arrive_expect_tx_elect(bar(C::kBarX), 2 * C::kTileBytes);
        for (int hf = 0; hf < C::kHalves; ++hf) {
          tma_load_3d_elect(x_smem(0) + hf * C::kSlabBytes, &tm_q, hf * 64, it.h, qrow, bar(C::kBarX));
          tma_load_3d_elect(x_smem(1) + hf * C::kSlabBytes, &tm_do, hf * 64, it.h, qrow, bar(C::kBarX));
        }
        ++xi;
        for (int t = 0; t < it.n_t; ++t) {
          const int row = it.sq.k0 + t * kTile;
          const int sk = kc % C::kKStages;
          if (kc >= C::kKStages &&
              !(ok = warp_wait_bar(bar(C::kBarKEmpty + sk), static_cast<uint32_t>(((kc / C::kKStages) & 1) ^ 1), wc)))
            break;
          mbar_arrive_expect_tx_elect(bar(C::kBarKFull + sk), C::kTileBytes);
          for (int hf = 0; hf < C::kHalves; ++hf)
            tma_load_3d_elect(k_smem(sk) + hf * C::kSlabBytes, &tm_k, hf * 64, it.hk, row, bar(C::kBarKFull + sk));
          ++kc;
          const int sv = vc % C::kVStages;
          if (vc >= C::kVStages &&
              !(ok = warp_wait_bar(bar(C::kBarVEmpty + sv), static_cast<uint32_t>(((vc / C::kVStages) & 1) ^ 1), wc)))
            break;
          mbar_arrive_expect_tx_elect(bar(C::kBarVFull + sv), C::kTileBytes);
          for (int hf = 0; hf < C::kHalves; ++hf)
            tma_load_3d_elect(v_smem(sv) + hf * C::kSlabBytes, &tm_v, hf * 64, it.hk, row, bar(C::kBarVFull + sv));
          ++vc;
        }
        if (!ok) break;
      }
      x = item_next(prm.sched, x, causal);
    }
    // let the copies this warp issued land before shared memory is released
    if (xi > 0) drain_wait(bar(C::kBarX), static_cast<uint32_t>((xi - 1) & 1));
    for (int s = 0; s < C::kKStages && s < kc; ++s) {
      const int last = s + ((kc - 1 - s) / C::kKStages) * C::kKStages;
      drain_wait(bar(C::kBarKFull + s), static_cast<uint32_t>((last / C::kKStages) & 1));
    }
    for (int s = 0; s < C::kVStages && s < vc; ++s) {
      const int last = s + ((vc - 1 - s) / C::kVStages) * C::kVStages;
      drain_wait(bar(C::kBarVFull + s), static_cast<uint32_t>((last / C::kVStages) & 1));
    }
  } else if (warp == kMma) {
    // ------------------------------------------------------------ MMA issue (converged warp)
    constexpr uint32_t idesc_score = instr_desc_f16(kTile, kTile, FP16, false);
    constexpr uint32_t idesc_acc = instr_desc_f16(kTile, D, FP16, true);
    constexpr uint64_t kTileStep = C::kTileBytes >> 4;
    const uint64_t q_desc = smem_desc_sw128(x_smem(0), 16, 1024);  // K-major
    const uint64_t do_desc = smem_desc_sw128(x_smem(1), 16, 1024);
    const uint64_t k_desc0 = smem_desc_sw128(k_smem(0), 16, 1024);
    const uint64_t v_desc0 = smem_desc_sw128(v_smem(0), 16, 1024);
    const uint64_t k_mn0 = smem_desc_sw128(k_smem(0), C::kSlabBytes, 1024);  // K_t as MN-major B of dQ += dS K
    // X Y^T into TMEM column `col`, K = D in steps of 16 (both operands K-major)
    auto issue_score = [&](uint64_t a, uint64_t bb, uint32_t col) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>(((kk / 4) * C::kSlabBytes + (kk % 4) * 32) >> 4);
        mma_ss_elect(tmem + col, a + off, bb + off, idesc_score, kk > 0 ? 1u : 0u);
      }
    };
    int kc = 0, vc = 0, tc = 0, xi = 0;  // K, V tiles, score tiles and items with work so far
    // S(t) = Q K_t^T into buffer (tc + t) % 2; dP(t) = dO V_t^T
    auto issue_s = [&](int t) {
      const int b = (tc + t) & 1;
      issue_score(q_desc, k_desc0 + static_cast<uint64_t>((kc + t) % C::kKStages) * kTileStep, C::kColS0 + 128 * b);
      mma_commit_elect(bar(C::kBarSFull + b));
    };
    auto issue_dp = [&](int t) {
      issue_score(do_desc, v_desc0 + static_cast<uint64_t>((vc + t) % C::kVStages) * kTileStep, C::kColDP);
      mma_commit_elect(bar(C::kBarDPFull));
    };
    auto wait_k = [&](int t) {
      return warp_wait_bar(bar(C::kBarKFull + (kc + t) % C::kKStages),
                           static_cast<uint32_t>(((kc + t) / C::kKStages) & 1), wc);
    };
    auto wait_v = [&](int t) {
      return warp_wait_bar(bar(C::kBarVFull + (vc + t) % C::kVStages),
                           static_cast<uint32_t>(((vc + t) / C::kVStages) & 1), wc);
    };
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int x = item_take(item_slots, full0, empty0, i, wc);
      if (x < 0) {
        ok = x == -1;
        break;
      }
      const ItemQ it = item_q(prm, x);
      const int n = it.n_t;
      if (n == 0) continue;
      ok = warp_wait_bar(bar(C::kBarX), static_cast<uint32_t>(xi & 1), wc) && wait_k(0);
      if (!ok) break;
      tc_fence_after();
      issue_s(0);
      if (!(ok = wait_v(0))) break;
      tc_fence_after();
      issue_dp(0);
      if (n == 1) mma_commit_elect(bar(C::kBarXEmpty));  // Q, dO of this item: last readers issued
      if (n > 1) {
        if (!(ok = wait_k(1))) break;
        tc_fence_after();
        issue_s(1);
      }
      for (int t = 0; ok && t < n; ++t) {
        const uint32_t ph = static_cast<uint32_t>((tc + t) & 1);
        // both warpgroups have read dP(t) and written dS(t) into its S buffer
        ok = warp_wait_bar(bar(C::kBarB), ph, wc) && warp_wait_bar(bar(C::kBarB + 1), ph, wc);
        if (!ok) break;
        tc_fence_after();
        mma_commit_elect(bar(C::kBarVEmpty + (vc + t) % C::kVStages));  // V_t: its reader dP(t) is done
        if (t + 1 < n) {
          if (!(ok = wait_v(t + 1))) break;
          tc_fence_after();
          issue_dp(t + 1);
          if (t + 1 == n - 1) mma_commit_elect(bar(C::kBarXEmpty));
        }
        // the item's first dQ product overwrites the accumulator: the previous
        // item's dQ must have been read out
        if (t == 0 && xi > 0) {
          if (!(ok = warp_wait_bar(bar(C::kBarAccEmpty), static_cast<uint32_t>((xi - 1) & 1), wc))) break;
          tc_fence_after();
        }
        // dQ += dS(t) K_t: A = dS pairs in its S buffer (warpgroup h: columns 64h ..), B = K_t MN-major
        const uint64_t kb = k_mn0 + static_cast<uint64_t>((kc + t) % C::kKStages) * kTileStep;
        const uint32_t a0 = C::kColS0 + 128 * ((tc + t) & 1);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          mma_ts_elect(tmem + C::kColAcc, tmem + a0 + 64 * (kk / 4) + 8 * (kk % 4),
                       kb + static_cast<uint64_t>(kk * (2048 >> 4)), idesc_acc, (t > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_elect(bar(C::kBarKEmpty + (kc + t) % C::kKStages));  // K_t: last reader issued
        if (t + 2 < n) {
          if (!(ok = wait_k(t + 2))) break;
          tc_fence_after();
          issue_s(t + 2);  // into the buffer of S(t), after dQ(t) has read dS(t) from it (in order)
        }
        if (t == n - 1) mma_commit_elect(bar(C::kBarDone));
      }
      kc += n;
      vc += n;
      tc += n;
      ++xi;
    }
    if (!ok) {
      mma_commit_elect(bar(C::kBarDrain));
      drain_wait(bar(C::kBarDrain), 0);
    }
  } else {
    // ------------------------------------------------------------ compute warpgroups (TMEM lane = row)
    const int wg = warp / 4;                  // column half of every score tile
    const int qd = warp % 4;                  // TMEM lane quadrant
    const int row = qd * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
    const float c = prm.scale_log2;
    int tc = 0, xi = 0;
    bool ok = true;
    // this thread's -LSE log2(e) and -D for item x (loaded ahead of use)
    auto row_values = [&](int x, float& nl, float& nd) {
      nl = 0.f;
      nd = 0.f;
      if (x < 0) return;
      const ItemQ it = item_q(prm, x);
      if (it.skip) return;
      const int64_t at = static_cast<int64_t>(it.bh) * prm.Npad + it.tile * kTile + row;
      nl = prm.ws_l[at];
      nd = prm.ws_d[at];
    };
    int x = item_take(item_slots, full0, empty0, 0, wc);
    float nl_row, nd_row;
    row_values(x, nl_row, nd_row);
    for (int i = 0; x >= 0; ++i) {
      const ItemQ it = item_q(prm, x);
      const int r_abs = it.tile * kTile + row;  // this thread's query
      if (!it.skip) {
        for (int t = 0; t < it.n_t; ++t) {
          const int T = tc + t;
          const int first_col = t * kTile + 64 * wg;  // first key of this warpgroup's half
          const uint32_t t_s = tmem + lane_base + C::kColS0 + 128 * (T & 1) + 64 * wg;
          // masked: the causal boundary cuts the tile (its last key is not seen by
          // the tile's first query), or the keys run out
          const bool masked =
              (causal && t * kTile + kTile - 1 > it.tile * kTile + it.sq.delta) || (t + 1) * kTile > it.sq.nk;
          ok = warp_wait_bar(bar(C::kBarSFull + (T & 1)), static_cast<uint32_t>((T >> 1) & 1), wc);
          if (!ok) break;
          tc_fence_after();
          float p[64];
          if (masked) {
            phase_a<FP16, false, true, false>(t_s, c, nl_row, nullptr, first_col, r_abs, it.sq.nk, causal,
                                              it.sq.delta, p);
          } else {
            phase_a<FP16, false, false, false>(t_s, c, nl_row, nullptr, first_col, r_abs, it.sq.nk, causal,
                                               it.sq.delta, p);
          }
          ok = warp_wait_bar(bar(C::kBarDPFull), static_cast<uint32_t>(T & 1), wc);
          if (!ok) break;
          tc_fence_after();
          // dS pairs over the first 32 columns of this half of S(t) (read above)
          phase_b<FP16, false>(tmem + lane_base + C::kColDP + 64 * wg, t_s, nd_row, nullptr, p);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(C::kBarB + wg));
        }
        if (!ok) break;
      } else if (!it.sq.ok && threadIdx.x == 0) {
        atomicOr(&g_status_word, 2u);  // inconsistent packed offsets
      }
      // the next item (published by now: this item's loads have all been
      // issued); its rows' values load while this item's dQ is written out
      const int nx = item_take(item_slots, full0, empty0, i + 1, wc);
      float nl_next, nd_next;
      row_values(nx, nl_next, nd_next);
      if (!it.skip) {
        if (it.n_t > 0 && !(ok = warp_wait_bar(bar(C::kBarDone), static_cast<uint32_t>(xi & 1), wc))) break;
        // warpgroup h writes dQ columns h D/2 .. (scaled); a tile whose queries
        // see no key at all gets 0. After the last read of the accumulator it
        // goes back to the MMA warp.
        const bool row_valid =
            r_abs < it.sq.nq && index_ok(static_cast<int64_t>(it.sq.q0) + r_abs < prm.total_q && it.h < prm.Hq);
        uint16_t* dst_row =
            prm.out0 + ((static_cast<int64_t>(it.sq.q0) + r_abs) * prm.Hq + it.h) * D + wg * (D / 2);
        const uint32_t acc = tmem + lane_base + C::kColAcc + wg * (D / 2);
        if (it.n_t > 0) tc_fence_after();
#pragma unroll
        for (int q = 0; q < D / 64; ++q) {
          uint32_t pk[16];
          if (it.n_t > 0) {
            uint32_t a[32];
            tmem_ld32(acc + q * 32, a);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 16; ++k)
              pk[k] = pack2<FP16>(__uint_as_float(a[2 * k]) * prm.scale, __uint_as_float(a[2 * k + 1]) * prm.scale);
            if (q == D / 64 - 1) {
              tc_fence_before();
              mbar_arrive(bar(C::kBarAccEmpty));
            }
          } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) pk[k] = 0u;
          }
          if (row_valid) store_row64(dst_row + q * 32, pk, prm.wide_stores != 0);
        }
        tc += it.n_t;
        if (it.n_t > 0) ++xi;
      }
      x = nx;
      nl_row = nl_next;
      nd_row = nd_next;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace bwd
}  // namespace fa
