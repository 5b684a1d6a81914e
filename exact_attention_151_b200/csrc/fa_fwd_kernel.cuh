// fa_fwd_kernel.cuh - the fused exact-attention forward kernel for sm_100a.
//
// What one CTA computes: O and LSE for a 256-row query block (two 128-row
// query tiles Q0, Q1) of one (batch, head), streaming over the visible
// 128-key tiles with an online softmax (running max and running sum per
// query row), so no N x N score or probability matrix reaches global memory:
//   * tiling Q / K / V and accumulating the softmax numerator and denominator
//     block by block: llmtrend.com FlashAttention page, "how it works";
//   * running max / running sum, rescaling the partial output: tuning handbook
//     ch. 3, "core idea" and the tiled routine in "engineering implementation";
//     jsqmd.com page, tiling + streaming;
//   * one fused kernel for QK^T -> softmax -> PV: jsqmd.com page, kernel fusion;
//   * K/V for the next tiles loaded while the current one is computed:
//     mlqm.cn FA1/FA2 comparison, section 2.2;
//   * work split over query blocks x batch x heads with K/V shared by the
//     block's rows: mlqm.cn section 2.1 (FA2 partition);
//   * causal attention skips future positions: handbook ch. 3, practical notes.
//
// Blackwell mapping (prior art on the pages targets Ampere; this is not it):
//   warp 9 (loader)    TMA 3-D tiled loads: Q0 and Q1 once, K_j and V_j into
//                      separate rings of 128B-swizzled shared-memory tiles;
//   warp 8 (MMA)       an elected lane of the converged warp issues tcgen05.mma in the order
//                        S0(j), PV1(j-1), S1(j), PV0(j)
//                      so that while one softmax warpgroup works on its
//                      scores the tensor cores serve the other query tile;
//                      S_i = Q_i K_j^T lands in TMEM (fp32), O_i += P_i V_j
//                      reads P_i from TMEM (16-bit) and V_j from shared memory;
//   warps 0-3 / 4-7    softmax warpgroup i for query tile i: one query row per
//                      thread (TMEM lane = row), so row max and row sum need
//                      no shuffles; writes P_i over the first half of S_i's
//                      columns; rescales O_i when its row max grew; finally
//                      normalises O_i and writes O and LSE.
// Because S_i(j) is issued after PV_i(j-1), the completion of S_i(j) implies
// that PV_i(j-1) has finished, so the O_i rescale needs no extra barrier.
// With packed heads and split-KV (the PAIR instantiation) both query tiles hold
// the same packed queries and each works through its own key range, so a CTA
// produces two partial results and both softmax warpgroups stay busy.
//
// Online-softmax bookkeeping (base 2, x = s * scale * log2(e)): m is only
// raised when a tile's max exceeds it by more than kRescaleThreshold, so
// P = 2^(x - m) stays below 2^threshold, which 16-bit P and fp32 sums hold
// easily; O and l always share the same m, so O / l and
// LSE = (m + log2 l) * ln 2 are exact up to rounding.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "sm100.cuh"

namespace fa {

using namespace sm100;

// Device status word: bit 0 set when some wait ran out, bit 1 for packed
// sequences with inconsistent offsets, bit 2 when a device-side index check of
// the checking build (FA_CHECKS) failed. Read and cleared by fa_status_sync. A
// static __device__ variable, so the library allocates nothing.
__device__ unsigned int g_status_word;

// Checking build (-DFA_CHECKS): every global store is preceded by a check that
// its index lies inside the tensor the host described; a failed check sets
// bit 2 of the status word and the store is skipped (no trap). In the normal
// build the check compiles to `true`.
__device__ __forceinline__ bool index_ok(bool in_range) {
#ifdef FA_CHECKS
  if (!in_range) atomicOr(&g_status_word, 4u);
  return in_range;
#else
  (void)in_range;
  return true;
#endif
}

constexpr int kTile = 128;        // query rows per tile = keys per tile = TMEM lanes
constexpr int kBlockRows = 256;   // query rows per CTA (two tiles)
constexpr int kHeadGroup = 16;    // heads whose query blocks are interleaved in the grid order
constexpr int kThreads = 384;     // 12 warps = 3 warpgroups
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;      // warps 10 and 11 only keep warpgroup 2 whole
// Registers per thread: the launch gives every thread kLaunchRegs (what ptxas
// allots for 384 threads); warpgroup 2 (MMA, loader) then gives registers back
// and the two softmax warpgroups take them. The shares must not exceed the
// launch pool, or the increase would wait forever:
constexpr uint32_t kLaunchRegs = 168;
constexpr uint32_t kSoftmaxRegs = 208;
constexpr uint32_t kControlRegs = 88;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * kLaunchRegs, "register split");
// The running max is raised only when a tile's max exceeds it by more than
// this (log2 units), so P = 2^(x - m) <= 2^15 stays inside fp16's range.
constexpr float kRescaleThreshold = 15.0f;
constexpr float kLn2 = 0.693147180559945309f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kMaxPolls = 1u << 28;
constexpr uint64_t kDrainLimitNs = 20ull * 1000 * 1000;

template <int D>
struct Cfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kHalves = D / 64;        // 64-element (128 B) column slabs per row
  static constexpr int kSlabBytes = 128 * 128;  // one slab: 128 rows x 128 B
  static constexpr int kTileBytes = kHalves * kSlabBytes;
  static constexpr int kKStages = (D == 128) ? 2 : 4;
  static constexpr int kVStages = (D == 128) ? 2 : 4;
  static constexpr int kQOff = 0;  // Q0 then Q1
  static constexpr int kKOff = kQOff + 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kVStages * kTileBytes;
  static constexpr int kBarQ = 0;
  static constexpr int kBarKFull = kBarQ + 1;
  static constexpr int kBarKEmpty = kBarKFull + kKStages;
  static constexpr int kBarVFull = kBarKEmpty + kKStages;
  static constexpr int kBarVEmpty = kBarVFull + kVStages;
  static constexpr int kBarSFull = kBarVEmpty + kVStages;  // [2]: S_i ready
  static constexpr int kBarPFull = kBarSFull + 2;          // [2][2]: half h of P_i written (128 arrivals)
  static constexpr int kBarOFinal = kBarPFull + 4;         // [2]: last PV_i done (single phase)
  static constexpr int kBarOStaged = kBarOFinal + 2;       // [2]: O_i staged in shared memory (128 arrivals)
  static constexpr int kBarDrain = kBarOStaged + 2;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base slot, abort flag
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + slack to align the base to 1024 B
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  // TMEM columns
  __host__ __device__ static constexpr uint32_t col_s(int i) { return static_cast<uint32_t>(i) * 128u; }
  __host__ __device__ static constexpr uint32_t col_o(int i) { return 256u + static_cast<uint32_t>(i * D); }
  static_assert(256 + 2 * D <= kTmemCols, "TMEM budget");
};

struct WaitCtl {
  volatile int* abort;
  uint64_t limit_ns;
};

// Bounded wait for the phase of `bar` with `parity`. Returns false if this
// CTA is aborting or the wait ran out (which starts the abort and records the
// timeout in the status word).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, WaitCtl w) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1; it < kMaxPolls; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*w.abort) return false;
    if ((it & 15u) == 0 && globaltimer_ns() - t0 > w.limit_ns) break;
  }
  *w.abort = 1;
  atomicOr(&g_status_word, 1u);
  return false;
}

// Short bounded wait used while tearing down (loads and MMAs in flight).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0; it < kMaxPolls; ++it) {
    if (mbar_try_wait(bar, parity)) return;
    if ((it & 15u) == 0 && globaltimer_ns() - t0 > kDrainLimitNs) return;
  }
}

// Warp-uniform wrapper: every lane polls; the warp proceeds only if all did.
__device__ __forceinline__ bool warp_wait_bar(uint32_t bar, uint32_t parity, WaitCtl w) {
  const bool ok = wait_bar(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

// Tile (query tile qt, key tile j) whose P is applied as P16 + (P - P16).
// Rows that see at most 128 keys keep all of them in key tile 0; for such
// rows a single 16-bit rounding of P weighs on the result about as much as
// the final rounding of O, so the residual is added with a second MMA pass.
// Causal: row i sees i + delta + 1 keys, so the tiles with such rows are those
// starting at or before row 127 - delta; otherwise it is every tile when the
// sequence has at most 128 keys. Elsewhere each row averages over more than
// 128 keys and the residual is negligible.
__device__ __forceinline__ bool split_p_tile(int qt, int j, int causal, int delta, int nk) {
  return j == 0 && (causal ? (qt * kTile <= kTile - 1 - delta) : (nk <= kTile));
}

// Max (MAX) or min of one row of 128 scores: three-input max in four
// independent chains.
template <bool MAX>
__device__ __forceinline__ float row_reduce(const float (&s)[kTile]) {
  auto r3 = [](float a, float b, float c) { return MAX ? max3f(a, b, c) : min3f(a, b, c); };
  float e0 = r3(s[0], s[1], s[2]);
  float e1 = r3(s[3], s[4], s[5]);
  float e2 = r3(s[6], s[7], s[8]);
  float e3 = r3(s[9], s[10], s[11]);
#pragma unroll
  for (int k = 12; k < kTile - 8; k += 8) {
    e0 = r3(e0, s[k], s[k + 1]);
    e1 = r3(e1, s[k + 2], s[k + 3]);
    e2 = r3(e2, s[k + 4], s[k + 5]);
    e3 = r3(e3, s[k + 6], s[k + 7]);
  }
  e0 = r3(e0, s[kTile - 4], s[kTile - 3]);
  e1 = r3(e1, s[kTile - 2], s[kTile - 1]);
  return r3(e0, e1, MAX ? fmaxf(e2, e3) : fminf(e2, e3));
}

// Half h of one row of one score tile (keys 64h .. 64h+63): p = 2^(s * c - m),
// packed to 16-bit pairs (key 2i in the low half of column i) and stored to
// TMEM columns 32h .. 32h+31 of S_i in two 16-column chunks; with SPLIT also
// the rounding residual p - p16 to columns 64 + 32h .. Returns the fp32 sum
// of p. Each score register dies once its pair is packed.
// Pairs of score columns whose exp2 runs on the FMA pipe (a Cody-Waite
// reduction and a polynomial) instead of the MUFU unit. At D = 64 a score
// tile carries half the tensor work of D = 128 for the same number of
// exponentials, so the exp unit alone would outlast the tensor cores: every
// fourth pair goes to the FMA pipe there. At D = 128 the exponentials fit the
// MUFU unit and the polynomial's extra instructions cost more than they save.
template <int D>
__device__ __forceinline__ constexpr bool fma_exp_pair(int pair) {
  return D == 64 && (pair & 3) == 3;
}

template <bool FP16, bool SPLIT, int HALF, int D>
__device__ __forceinline__ float softmax_exp_half(const float (&s)[kTile], float c, float m, uint32_t s_col) {
  const float2 c2 = make_float2(c, c);
  const float2 nm2 = make_float2(-m, -m);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int chunk = 0; chunk < 2; ++chunk) {
    uint32_t pk[16];
    uint32_t lo[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int pr = HALF * 32 + chunk * 16 + q;  // pair index in the row
      const float2 x = ffma2(make_float2(s[2 * pr], s[2 * pr + 1]), c2, nm2);
      const float2 p = fma_exp_pair<D>(pr) ? exp2_poly2(x) : make_float2(ex2_approx(x.x), ex2_approx(x.y));
      if (q & 1) {
        acc1 = fadd2(acc1, p);
      } else {
        acc0 = fadd2(acc0, p);
      }
      pk[q] = pack2<FP16>(p.x, p.y);
      if constexpr (SPLIT) {
        const float2 hf = unpack2<FP16>(pk[q]);
        lo[q] = pack2<FP16>(p.x - hf.x, p.y - hf.y);
      }
    }
    tmem_st16(s_col + HALF * 32 + chunk * 16, pk);
    if constexpr (SPLIT) tmem_st16(s_col + 64 + HALF * 32 + chunk * 16, lo);
  }
  const float2 acc = fadd2(acc0, acc1);
  return acc.x + acc.y;
}

// Chunk CH (0..3) of one row of one score tile (keys 32 CH .. 32 CH + 31, i.e.
// pairs 16 CH .. 16 CH + 15): p = 2^(s * c - m) packed to 16-bit pairs into
// pk (the caller stores them to TMEM columns 16 CH ..); returns the fp32 sum
// of p as two partial sums. Nothing is stored, so the caller decides where the
// TMEM stores and hand-offs go.
template <bool FP16, int CH>
__device__ __forceinline__ float2 softmax_exp_chunk(const float (&s)[kTile], float c, float m, uint32_t (&pk)[16]) {
  const float2 c2 = make_float2(c, c);
  const float2 nm2 = make_float2(-m, -m);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    const int pr = CH * 16 + q;  // pair index in the row
    const float2 x = ffma2(make_float2(s[2 * pr], s[2 * pr + 1]), c2, nm2);
    const float2 p = make_float2(ex2_approx(x.x), ex2_approx(x.y));
    if (q & 1) {
      acc1 = fadd2(acc1, p);
    } else {
      acc0 = fadd2(acc0, p);
    }
    pk[q] = pack2<FP16>(p.x, p.y);
  }
  return fadd2(acc0, acc1);
}

// O row *= alpha in TMEM (warp-collective; D columns from o_col).
template <int D>
__device__ __forceinline__ void rescale_o(uint32_t o_col, float alpha) {
#pragma unroll
  for (int q = 0; q < D / 32; ++q) {
    uint32_t o[32];
    tmem_ld32(o_col + q * 32, o);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 32; k += 2) {
      const float2 v = fmul2(make_float2(__uint_as_float(o[k]), __uint_as_float(o[k + 1])), make_float2(alpha, alpha));
      o[k] = __float_as_uint(v.x);
      o[k + 1] = __float_as_uint(v.y);
    }
    tmem_st32(o_col + q * 32, o);
  }
}

// Problem description passed by value.
struct Params {
  uint16_t* out;        // [total_q, Hq, D]
  float* lse;           // dense: [B, Hq, Nq]; packed: [Hq, total_q]
  const int* cu_q;      // packed sequences: B+1 query row offsets (device memory); dense: null
  const int* cu_k;      // packed sequences: B+1 key row offsets
  int Nq, Nk;           // dense sequence lengths
  int total_q, total_k; // rows of q/o and of k/v
  int Hq, Hkv;          // query heads, key/value heads (Hq % Hkv == 0)
  int BH;               // B * Hq
  int max_nq;           // upper bound of every query length (sizes the grid)
  int n_blocks;         // ceil(max_nq / 256)
  float scale_log2;
  int causal;           // key j visible to query i iff j <= i + nk - nq (bottom-right aligned)
  // Split-KV (n_splits > 1, dense shapes only): key range s covers key tiles
  // [s * split_tiles, (s + 1) * split_tiles) and writes its own normalised O
  // and LSE, in fp32, to part_o [n_splits, B, Hq, Nq, D] and part_lse
  // [n_splits, B, Hq, Nq]; a separate kernel merges the splits.
  int n_splits;
  int split_tiles;
  float* part_o;
  float* part_lse;
  unsigned long long wait_limit_ns;
  int withhold_v_load;
  // Packed heads (dense shapes with Nq * G <= 128, G = Hq / Hkv > 1): one work
  // item per (batch, key/value head); its single query tile holds the G query
  // heads sharing that K/V head for every query position, row n G + g = query
  // n of head hk G + g (one TMA box of (64, G, Nq)). BH then counts B * Hkv
  // items and BHq = B * Hq query heads. 0: off.
  int pack_g;
  int BHq;
};

// PAIR (paired split-KV, for packed heads with n_splits > 1): the second query
// tile holds the same packed queries as the first, and CTA split c computes the
// partial results of key ranges 2c (tile 0) and 2c + 1 (tile 1) side by side,
// each tile with its own K and V tiles. A template parameter, so that the
// unpaired MMA issue loop carries none of its bookkeeping (each instruction of
// the issuing warp is tensor-pipe time).
template <int D, bool FP16, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const Params prm) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto q_smem = [&](int i) { return sbase + C::kQOff + i * C::kTileBytes; };
  auto k_smem = [&](int s) { return sbase + C::kKOff + s * C::kTileBytes; };
  auto v_smem = [&](int s) { return sbase + C::kVOff + s * C::kTileBytes; };
  auto bar = [&](int i) { return sbase + C::kBarOff + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int causal = prm.causal;

  // Split-KV index is the slowest-varying part of the block index.
  const int split = static_cast<int>(blockIdx.x) / (prm.BH * prm.n_blocks);
  const int xblk = static_cast<int>(blockIdx.x) - split * (prm.BH * prm.n_blocks);
  int bh, level;
  {
    // Causal: heads in groups of kHeadGroup; inside a group, query-block level
    // by level across the group's heads, heaviest first. The group's K/V stay
    // in L2 while its CTAs run, and the last CTAs to start are the lightest.
    const int per_group = kHeadGroup * prm.n_blocks;
    const int full_groups = prm.BH / kHeadGroup;
    const int x = xblk;
    int g, hg, within;
    if (x < full_groups * per_group) {
      g = x / per_group;
      hg = kHeadGroup;
      within = x % per_group;
    } else {
      g = full_groups;
      hg = prm.BH - full_groups * kHeadGroup;
      within = x - full_groups * per_group;
    }
    level = within / hg;
    bh = g * kHeadGroup + within % hg;
  }
  if (!causal) {
    // equal work per block: keep all blocks of a head adjacent (K/V shared in L2)
    bh = xblk / prm.n_blocks;
    level = xblk % prm.n_blocks;
  }
  const int mb = causal ? (prm.n_blocks - 1 - level) : level;
  const int pg = prm.pack_g;
  const int b = pg ? bh / prm.Hkv : bh / prm.Hq;
  const int h = pg ? (bh % prm.Hkv) * pg : bh % prm.Hq;    // (first) query head
  const int hk = pg ? bh % prm.Hkv : h / (prm.Hq / prm.Hkv);  // key/value head
  // This sequence's rows: queries q0 .. q0+nq-1, keys k0 .. k0+nk-1.
  int q0, nq, k0, nk;
  if (prm.cu_q != nullptr) {
    q0 = prm.cu_q[b];
    nq = prm.cu_q[b + 1] - q0;
    k0 = prm.cu_k[b];
    nk = prm.cu_k[b + 1] - k0;
    const bool bad = q0 < 0 || nq < 0 || nq > prm.max_nq || static_cast<int64_t>(q0) + nq > prm.total_q || k0 < 0 ||
                     nk < 0 || static_cast<int64_t>(k0) + nk > prm.total_k;
    if (bad) {  // inconsistent offsets: report, touch nothing
      if (threadIdx.x == 0) atomicOr(&g_status_word, 2u);
      return;
    }
  } else {
    q0 = b * prm.Nq;
    nq = prm.Nq;
    k0 = b * prm.Nk;
    nk = prm.Nk;
  }
  if (mb * kBlockRows >= nq) return;  // block past the end of this sequence
  const int n_qt = (nq + kTile - 1) / kTile;
  const int n_kt = (nk + kTile - 1) / kTile;
  const int delta = nk - nq;  // causal offset: query i sees keys j <= i + delta
  const int qt0 = 2 * mb;
  const int qt1 = 2 * mb + 1;
  constexpr bool pair = PAIR;
  // partial-result slot (split-KV) of tile 0; tile 1 takes the next one when paired
  const int slot0 = pair ? 2 * split : split;
  const bool q1_valid = pair ? slot0 + 1 < prm.n_splits : (!pg && qt1 < n_qt);
  // smallest and largest query index held by query tile qt (packed heads:
  // the first and the last query)
  auto q_min = [&](int qt) -> int { return pg ? 0 : qt * kTile; };
  auto q_max = [&](int qt) -> int { return pg ? nq - 1 : qt * kTile + kTile - 1; };
  // last key tile holding a key visible to some row of query tile qt (-1: none)
  auto last_key_tile = [&](int qt) -> int {
    if (nk == 0) return -1;
    if (!causal) return n_kt - 1;
    const int last_key = q_max(qt) + delta;
    if (last_key < 0) return -1;
    return min(n_kt - 1, last_key / kTile);
  };
  // Key tiles of query tile i: jb_i .. je_i - 1 (all of them unless split-KV;
  // one range for both tiles unless paired). Tile indices below are relative to
  // jb_i; last_i is the last tile (relative) with a key visible to some row of
  // query tile i, -1 if none.
  const int jb0 = slot0 * prm.split_tiles;
  const int jb1 = pair ? jb0 + prm.split_tiles : jb0;
  auto last_rel = [&](int qt, int jb) -> int {
    const int je = prm.n_splits > 1 ? min(n_kt, jb + prm.split_tiles) : n_kt;
    const int t = min(last_key_tile(qt), je - 1);
    return t < jb ? -1 : t - jb;
  };
  const int last0 = last_rel(qt0, jb0);
  const int last1 = q1_valid ? last_rel(pair ? qt0 : qt1, jb1) : -1;
  const int n_kv = (last1 > last0 ? last1 : last0) + 1;
  // K and V tiles go through their rings as items, in load order. Unpaired,
  // item j is key tile jb + j, shared by both query tiles. Paired (last1 <=
  // last0 there: tile 1's range starts later), items alternate tile 0 and tile 1
  // while both have tiles, then tile 0's remaining ones follow.
  const int n_items = pair ? (last0 + 1) + (last1 + 1) : n_kv;
  auto item_of = [&](int i, int j) -> int { return !pair ? j : (j <= last1 ? 2 * j + i : last1 + 1 + j); };
  auto item_key_tile = [&](int u) -> int {  // absolute key tile of item u
    if (!pair) return jb0 + u;
    if (u < 2 * (last1 + 1)) return ((u & 1) ? jb1 : jb0) + (u >> 1);
    return jb0 + (u - (last1 + 1));
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(C::kBarQ), 1);
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
      mbar_init(bar(C::kBarPFull + 2 * i), 128);
      mbar_init(bar(C::kBarPFull + 2 * i + 1), 128);
      mbar_init(bar(C::kBarOFinal + i), 1);
      mbar_init(bar(C::kBarOStaged + i), 128);
    }
    mbar_init(bar(C::kBarDrain), 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, prm.wait_limit_ns};

  if (warp >= 8) {
    regs_decrease<kControlRegs>();
    if (warp == kLoadWarp) {
    // ------------------------------------------------------------ loader
    // The whole warp runs this loop (converged); one elected lane issues each
    // barrier arm and TMA copy. (A second loader warp for V measured slower: one
    // more polling warp shares a sub-partition with two softmax warps.)
    {
      if (lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
      }
      __syncwarp();
      if (pg) {
        // packed heads: one (64, G, Nq) box per slab fills rows 0 .. G Nq - 1
        // (into both query tiles when paired)
        const int nt = pair ? 2 : 1;
        mbar_arrive_expect_tx_elect(bar(C::kBarQ), nt * C::kHalves * pg * nq * 128);
        for (int i = 0; i < nt; ++i)
          for (int hf = 0; hf < C::kHalves; ++hf)
            tma_load_3d_elect(q_smem(i) + hf * C::kSlabBytes, &tm_q, hf * 64, h, q0, bar(C::kBarQ));
      } else {
        mbar_arrive_expect_tx_elect(bar(C::kBarQ), (q1_valid ? 2 : 1) * C::kTileBytes);
        for (int i = 0; i < (q1_valid ? 2 : 1); ++i)
          for (int hf = 0; hf < C::kHalves; ++hf)
            tma_load_3d_elect(q_smem(i) + hf * C::kSlabBytes, &tm_q, hf * 64, h, q0 + (qt0 + i) * kTile, bar(C::kBarQ));
      }
      const bool withhold = prm.withhold_v_load && blockIdx.x == 0;  // V item 0 of CTA 0
      int nk_issued = 0, nv_issued = 0;  // K and V items handled
      for (int u = 0; u < n_items; ++u) {
        const int key_row = k0 + item_key_tile(u) * kTile;
        const int sk = u % C::kKStages;
        if (u >= C::kKStages &&
            !warp_wait_bar(bar(C::kBarKEmpty + sk), static_cast<uint32_t>(((u / C::kKStages) & 1) ^ 1), wc))
          break;
        mbar_arrive_expect_tx_elect(bar(C::kBarKFull + sk), C::kTileBytes);
        for (int hf = 0; hf < C::kHalves; ++hf)
          tma_load_3d_elect(k_smem(sk) + hf * C::kSlabBytes, &tm_k, hf * 64, hk, key_row, bar(C::kBarKFull + sk));
        nk_issued = u + 1;
        const int sv = u % C::kVStages;
        if (u >= C::kVStages &&
            !warp_wait_bar(bar(C::kBarVEmpty + sv), static_cast<uint32_t>(((u / C::kVStages) & 1) ^ 1), wc))
          break;
        if (!(withhold && u == 0)) {
          mbar_arrive_expect_tx_elect(bar(C::kBarVFull + sv), C::kTileBytes);
          for (int hf = 0; hf < C::kHalves; ++hf)
            tma_load_3d_elect(v_smem(sv) + hf * C::kSlabBytes, &tm_v, hf * 64, hk, key_row, bar(C::kBarVFull + sv));
        }
        nv_issued = u + 1;
      }
      // Let every load this thread issued land before shared memory is
      // released (immediate in a normal run, where all were consumed): for
      // each stage, wait for the phase of its last arming.
      drain_wait(bar(C::kBarQ), 0);
      for (int st = 0; st < C::kKStages && st < nk_issued; ++st) {
        const int ul = st + ((nk_issued - 1 - st) / C::kKStages) * C::kKStages;
        drain_wait(bar(C::kBarKFull + st), static_cast<uint32_t>((ul / C::kKStages) & 1));
      }
      for (int st = 0; st < C::kVStages && st < nv_issued; ++st) {
        const int ul = st + ((nv_issued - 1 - st) / C::kVStages) * C::kVStages;
        if (!(withhold && ul == 0)) drain_wait(bar(C::kBarVFull + st), static_cast<uint32_t>((ul / C::kVStages) & 1));
      }
    }
    __syncwarp();
    } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop (converged, descriptors in uniform
    // registers); one elected lane issues each tcgen05.mma and commit.
    {
      constexpr uint32_t idesc_qk = instr_desc_f16(kTile, kTile, FP16, false);
      constexpr uint32_t idesc_pv = instr_desc_f16(kTile, D, FP16, true);
      // Shared-memory descriptors are built once; a tile, stage or K step is
      // reached by adding its byte offset / 16 to the start-address field
      // (bits 0-13; shared addresses stay below 2^18, so nothing carries out).
      // Keeping per-MMA work to one add lets issue keep up with the tensor pipe.
      const uint64_t q_desc0 = smem_desc_sw128(q_smem(0), 16, 1024);
      const uint64_t k_desc0 = smem_desc_sw128(k_smem(0), 16, 1024);
      const uint64_t v_desc0 = smem_desc_sw128(v_smem(0), C::kSlabBytes, 1024);
      constexpr uint64_t kTileStep = C::kTileBytes >> 4;
      // S_i(j) = Q_i K_j^T  (K-major A and B, K = D in steps of 16)
      auto issue_s = [&](int i, int sk) {
        const uint64_t qa = q_desc0 + static_cast<uint64_t>(i) * kTileStep;
        const uint64_t kb = k_desc0 + static_cast<uint64_t>(sk) * kTileStep;
        const uint32_t d_tmem = tmem + C::col_s(i);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk / 4) * C::kSlabBytes + (kk % 4) * 32) >> 4);
          mma_ss_elect(d_tmem, qa + off, kb + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit_elect(bar(C::kBarSFull + i));
      };
      // O_i += P_i(j) V_j for keys 64h .. 64h+63 (P from TMEM, V MN-major,
      // K in steps of 16); the split tile adds the residual pass.
      auto issue_pv_half = [&](int i, int j, int sv, bool split, int h) {
        const uint64_t vb = v_desc0 + static_cast<uint64_t>(sv) * kTileStep;
        const uint32_t o_tmem = tmem + C::col_o(i);
        const uint32_t p_tmem = tmem + C::col_s(i);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int kk = 4 * h + q;
          mma_ts_elect(o_tmem, p_tmem + kk * 8, vb + static_cast<uint64_t>(kk * (2048 >> 4)), idesc_pv,
                       (j > 0 || kk > 0) ? 1u : 0u);
        }
        if (split) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int kk = 4 * h + q;
            mma_ts_elect(o_tmem, p_tmem + 64 + kk * 8, vb + static_cast<uint64_t>(kk * (2048 >> 4)), idesc_pv, 1u);
          }
        }
      };
      // Both halves of PV_i(j) with the V item u: each waits for its half of P.
      // V is waited for first (with need_v; false when this warp has already
      // observed V item u): it is normally resident by now, and P, which is
      // not, then ends the wait with nothing left to check behind it.
      auto issue_pv = [&](int i, int j, int u, bool split, bool need_v) -> bool {
        const int sv = u % C::kVStages;
        if ((need_v && !warp_wait_bar(bar(C::kBarVFull + sv), static_cast<uint32_t>((u / C::kVStages) & 1), wc)) ||
            !warp_wait_bar(bar(C::kBarPFull + 2 * i), static_cast<uint32_t>(j & 1), wc))
          return false;
        tc_fence_after();
        issue_pv_half(i, j, sv, split, 0);
        if (!warp_wait_bar(bar(C::kBarPFull + 2 * i + 1), static_cast<uint32_t>(j & 1), wc)) return false;
        tc_fence_after();
        issue_pv_half(i, j, sv, split, 1);
        return true;
      };
      const bool split0 = jb0 == 0 && split_p_tile(qt0, 0, causal, delta, nk);
      const bool split1 = jb1 == 0 && split_p_tile(pair ? qt0 : qt1, 0, causal, delta, nk);
      // wait for K item u; false if the CTA is aborting
      auto wait_k = [&](int u) -> bool {
        if (!warp_wait_bar(bar(C::kBarKFull + u % C::kKStages), static_cast<uint32_t>((u / C::kKStages) & 1), wc))
          return false;
        tc_fence_after();
        return true;
      };
      // Every wait between two MMA groups leaves the tensor pipe idle while it
      // runs, even one already satisfied (an mbarrier poll with its warp vote
      // takes longer than the one MMA the pipe still holds). So, unpaired,
      // the waits that are normally satisfied are taken where the warp would
      // block anyway, on P: V item j before PV0(j)'s P (PV1(j) then needs no
      // V wait: this warp has observed it), and K item j+1 probed there too
      // (k_seen), so that PV0(j) -> S0(j+1) runs with no wait between.
      bool ok = warp_wait_bar(bar(C::kBarQ), 0, wc);
      bool k_seen = false;  // K item of the next S0 already observed
      for (int j = 0; ok && j <= n_kv; ++j) {
        if (j < n_kv && (j <= last0 || !pair)) {
          // S0(j); unpaired, K item j also serves S1(j) and is waited for here
          const int u = item_of(0, j);
          if (k_seen) {
            tc_fence_after();
          } else if (!(ok = wait_k(u))) {
            break;
          }
          k_seen = false;
          if (j <= last0) issue_s(0, u % C::kKStages);
          if (pair && u + C::kKStages < n_items) mma_commit_elect(bar(C::kBarKEmpty + u % C::kKStages));
        }
        if (j >= 1 && j - 1 <= last1) {
          // PV1(j-1): the tensor cores work on it while softmax 0 handles S0(j)
          const int jp = j - 1, u = item_of(1, jp);
          // unpaired: PV0(jp) observed V item jp unless jp > last0
          ok = issue_pv(1, jp, u, split1 && jp == 0, pair || jp > last0);
          if (!ok) break;
          if (jp == last1) mma_commit_elect(bar(C::kBarOFinal + 1));
          // unpaired: PV1 is V_jp's last reader; paired: its only one
          if (u + C::kVStages < n_items) mma_commit_elect(bar(C::kBarVEmpty + u % C::kVStages));
        }
        if (j < n_kv) {
          if (j <= last1) {
            const int u = item_of(1, j);
            if (pair && !(ok = wait_k(u))) break;
            issue_s(1, u % C::kKStages);
            if (pair && u + C::kKStages < n_items) mma_commit_elect(bar(C::kBarKEmpty + u % C::kKStages));
          }
          // unpaired: K_j's last reader has been issued
          if (!pair && j + C::kKStages < n_kv) mma_commit_elect(bar(C::kBarKEmpty + j % C::kKStages));
          if (j <= last0) {
            const int u = item_of(0, j);
            if (!pair) {
              // V item j, then a poll of K item j+1, before PV0(j)'s P wait
              if (!(ok = warp_wait_bar(bar(C::kBarVFull + u % C::kVStages),
                                       static_cast<uint32_t>((u / C::kVStages) & 1), wc)))
                break;
              if (j + 1 < n_kv)
                k_seen = __all_sync(0xffffffffu, mbar_test_wait(bar(C::kBarKFull + (j + 1) % C::kKStages),
                                                                static_cast<uint32_t>(((j + 1) / C::kKStages) & 1)));
            }
            ok = issue_pv(0, j, u, split0 && j == 0, pair);
            if (!ok) break;
            if (j == last0) mma_commit_elect(bar(C::kBarOFinal + 0));
            if ((pair || j > last1) && u + C::kVStages < n_items) mma_commit_elect(bar(C::kBarVEmpty + u % C::kVStages));
          }
        }
      }
      if (!ok) {
        mma_commit_elect(bar(C::kBarDrain));
        drain_wait(bar(C::kBarDrain), 0);
      }
    }
    __syncwarp();
    }
  } else {
    regs_increase<kSoftmaxRegs>();
    // ------------------------------------------------------------ softmax warpgroups
    const int wg = warp / 4;              // query tile of this warpgroup
    const int qt = pair ? qt0 : qt0 + wg;  // paired: both tiles hold the same queries
    const int last = wg == 0 ? last0 : last1;
    const int jb = wg == 0 ? jb0 : jb1;   // first key tile of this tile's range
    const int quarter = warp % 4;         // TMEM lane quarter this warp may access
    const int row = quarter * 32 + lane;
    // this row's query index and head (packed heads: row = n G + g)
    const int qi = pg ? row / pg : qt * kTile + row;
    const int hq = pg ? h + row % pg : h;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_col = tmem + lane_base + C::col_s(wg);
    const uint32_t o_col = tmem + lane_base + C::col_o(wg);
    const float c = prm.scale_log2;
    const bool c_pos = c > 0.f;  // host guarantees c != 0
    const float fill = c_pos ? -INFINITY : INFINITY;  // masked score: weight 2^-inf = 0
    float m_used = -INFINITY;
    float l_sum = 0.f;
    bool ok = true;
    // packed heads: a warp whose 32 rows are all past the G Nq real ones only
    // keeps the hand-offs (its rows' O is never stored)
    const bool warp_idle = pg && quarter * 32 >= pg * nq;
    // Speculate (exponentials before the tile max; D = 128 only: at D = 64 the
    // exp unit, not the max chain, bounds a tile) until a tile's max outgrows
    // the threshold once: rows whose max keeps growing (very large logits)
    // then take the max-first path for the rest of the item. Warp-uniform.
    bool speculate = D == 128;
    for (int j = 0; j <= last; ++j) {
      ok = warp_wait_bar(bar(C::kBarSFull + wg), static_cast<uint32_t>(j & 1), wc);
      if (!ok) break;
      tc_fence_after();
      if (warp_idle) {
        tc_fence_before();
        mbar_arrive(bar(C::kBarPFull + 2 * wg));
        mbar_arrive(bar(C::kBarPFull + 2 * wg + 1));
        continue;
      }
      const int kbase = (jb + j) * kTile;
      // masking is needed when some row of the tile sees only part of it: the
      // tile runs past the keys, or past the first row's last visible key
      const bool masked = kbase + kTile > nk || (causal && kbase + kTile - 1 > q_min(qt) + delta);
      // last visible column of this row in this tile (may be < 0: none)
      const int lastcol = (causal ? min(nk - 1, qi + delta) : (nk - 1)) - kbase;
      if (j > 0 && speculate) {
        // Fast path for every tile after the first: the running max m_used is
        // known, and as long as this tile's max exceeds it by at most
        // kRescaleThreshold, P = 2^(x - m_used) is exactly what the lazy
        // rescale uses. So the first half's exponentials start at once and the
        // tile max (an independent chain) runs alongside them. The first
        // half's P stays in registers until the max is checked: if the max
        // grew past the threshold (rare after the first tile) nothing has been
        // written, and the tile is redone below from the scores still in TMEM.
        float sf[kTile];
        {
          uint32_t r[4][32];
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_ld32(s_col + q * 32, r[q]);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < kTile; ++k) sf[k] = __uint_as_float(r[k / 32][k % 32]);
        }
        if (masked) {
#pragma unroll
          for (int k = 0; k < kTile; ++k) sf[k] = (k <= lastcol) ? sf[k] : fill;
        }
        const float m_raw = c_pos ? row_reduce<true>(sf) : row_reduce<false>(sf);
        uint32_t pk0[16], pk1[16];
        float2 acc = softmax_exp_chunk<FP16, 0>(sf, c, m_used, pk0);
        acc = fadd2(acc, softmax_exp_chunk<FP16, 1>(sf, c, m_used, pk1));
        if (!__any_sync(0xffffffffu, m_raw * c > m_used + kRescaleThreshold)) {
          tmem_st16(s_col, pk0);
          tmem_st16(s_col + 16, pk1);
          // the second half's first chunk is computed while those stores complete
          uint32_t pk2[16];
          float2 acc2 = softmax_exp_chunk<FP16, 2>(sf, c, m_used, pk2);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(C::kBarPFull + 2 * wg));
          tmem_st16(s_col + 32, pk2);
          acc2 = fadd2(acc2, softmax_exp_chunk<FP16, 3>(sf, c, m_used, pk2));
          tmem_st16(s_col + 48, pk2);
          const float2 tot = fadd2(acc, acc2);
          l_sum += tot.x + tot.y;
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(C::kBarPFull + 2 * wg + 1));
          continue;
        }
        speculate = false;  // the max grew: this warp's later tiles start with the max
      }
      // First tile of the range (the running max starts here), a tile whose
      // max grew past the threshold, or any tile after one: the tile max
      // comes first.
      float s[kTile];
      {
        uint32_t r[4][32];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld32(s_col + q * 32, r[q]);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < kTile; ++k) s[k] = __uint_as_float(r[k / 32][k % 32]);
      }
      if (masked) {
#pragma unroll
        for (int k = 0; k < kTile; ++k) s[k] = (k <= lastcol) ? s[k] : fill;
      }
      // tile max of x = s * c: c * max(s) for c > 0, c * min(s) for c < 0 (exact under rounding)
      const float m_tile = (c_pos ? row_reduce<true>(s) : row_reduce<false>(s)) * c;
      const float m_new = fmaxf(m_used, m_tile);
      const bool rescale = m_new > m_used + kRescaleThreshold;  // always true on the first tile
      float alpha = 1.f;
      if (rescale) {
        alpha = ex2_approx(m_used - m_new);  // 0 on the first tile (m_used = -inf)
        l_sum *= alpha;
        m_used = m_new;
      }
      // O_i holds the sum up to tile j-1 under the old max; PV_i(j-1) has
      // completed because S_i(j) was issued after it and has completed. TMEM
      // access is warp-collective: the whole warp rescales, others by 1.
      if (j > 0 && __any_sync(0xffffffffu, rescale)) rescale_o<D>(o_col, alpha);
      // P = 2^(s * c - m) over the first 64 columns of S_i, published in two
      // halves (keys 0-63, 64-127) so the PV MMA can start on the first.
      float psum;
      if (split_p_tile(qt, jb + j, causal, delta, nk)) {
        psum = softmax_exp_half<FP16, true, 0, D>(s, c, m_used, s_col);
      } else {
        psum = softmax_exp_half<FP16, false, 0, D>(s, c, m_used, s_col);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::kBarPFull + 2 * wg));
      if (split_p_tile(qt, jb + j, causal, delta, nk)) {
        psum += softmax_exp_half<FP16, true, 1, D>(s, c, m_used, s_col);
      } else {
        psum += softmax_exp_half<FP16, false, 1, D>(s, c, m_used, s_col);
      }
      l_sum += psum;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::kBarPFull + 2 * wg + 1));
    }
    if (last >= 0 && ok) ok = warp_wait_bar(bar(C::kBarOFinal + wg), 0, wc);
    // Epilogue. A row with no visible key (bottom-right causal with nq > nk,
    // or nk == 0; with split-KV: none in this split's key range) gets O = 0
    // and LSE = -inf, whatever its TMEM lanes hold.
    const bool splitkv = prm.n_splits > 1;
    const int row_last_key = causal ? min(nk - 1, qi + delta) : nk - 1;
    const bool row_valid = (wg == 0 || q1_valid) && qi < nq && (!pg || row < pg * nq);
    const bool row_has_keys = row_last_key >= 0 && (!splitkv || row_last_key >= jb * kTile);
    if (splitkv) {
      // fp32 partial result of this key range (normalised by its own sum)
      const int64_t prow = (static_cast<int64_t>(slot0 + (pair ? wg : 0)) * prm.BHq + static_cast<int64_t>(b) * prm.Hq + hq) * prm.Nq + qi;
      float* orow = prm.part_o + prow * D;
      const bool prow_ok =
          !row_valid || index_ok(prow >= 0 && prow < static_cast<int64_t>(prm.n_splits) * prm.BHq * prm.Nq);
      if (last >= 0 && ok) {
        tc_fence_after();
        const float inv_l = row_has_keys ? 1.f / l_sum : 0.f;
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
          uint32_t o[32];
          tmem_ld32(o_col + q * 32, o);
          tmem_wait_ld();
          if (row_valid && prow_ok) {
            uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const float2 a = fmul2(make_float2(__uint_as_float(o[4 * k]), __uint_as_float(o[4 * k + 1])),
                                     make_float2(inv_l, inv_l));
              const float2 c2 = fmul2(make_float2(__uint_as_float(o[4 * k + 2]), __uint_as_float(o[4 * k + 3])),
                                      make_float2(inv_l, inv_l));
              dst[k] = row_has_keys ? make_uint4(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(c2.x),
                                                 __float_as_uint(c2.y))
                                    : make_uint4(0u, 0u, 0u, 0u);
            }
          }
        }
        if (row_valid && prow_ok) prm.part_lse[prow] = row_has_keys ? (m_used + lg2_approx(l_sum)) * kLn2 : -INFINITY;
      } else if (last < 0 && row_valid && prow_ok) {
        uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
        for (int k = 0; k < D / 4; ++k) dst[k] = make_uint4(0u, 0u, 0u, 0u);
        prm.part_lse[prow] = -INFINITY;
      } else if (row_valid && prow_ok) {
        // a wait ran out: mark this range's partial result invalid so the merge
        // yields NaN rather than combining what an earlier call left behind
        prm.part_lse[prow] = __int_as_float(0x7fc00000);
      }
    } else {
      uint16_t* orow = prm.out + (static_cast<int64_t>(q0 + qi) * prm.Hq + hq) * D;
      const int64_t lse_idx = prm.cu_q != nullptr ? static_cast<int64_t>(hq) * prm.total_q + q0 + qi
                                                  : (static_cast<int64_t>(b) * prm.Hq + hq) * prm.Nq + qi;
      float* lse_at = prm.lse + lse_idx;
      // dense: lse is [B, Hq, Nq]; packed: [Hq, total_q]
      const int64_t lse_len = prm.cu_q != nullptr ? static_cast<int64_t>(prm.Hq) * prm.total_q
                                                  : static_cast<int64_t>(prm.BHq) * prm.Nq;
      const bool out_ok = !row_valid || index_ok(q0 + qi >= 0 && q0 + qi < prm.total_q && hq >= 0 && hq < prm.Hq &&
                                                 lse_idx >= 0 && lse_idx < lse_len);
      // A full dense tile leaves through one TMA store per 64-column slab,
      // staged in this warpgroup's Q buffer (free: every S_i has completed,
      // and OFinal_i has been seen) in the 128B-swizzled layout of the map.
      const bool tma_out = prm.cu_q == nullptr && !pg && (qt + 1) * kTile <= nq;
      if (last >= 0 && ok) {
        tc_fence_after();
        const float inv_l = row_has_keys ? 1.f / l_sum : 0.f;
        uint8_t* qbuf = smem + C::kQOff + wg * C::kTileBytes;
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
          uint32_t o[32];
          tmem_ld32(o_col + q * 32, o);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const float2 v = fmul2(make_float2(__uint_as_float(o[2 * k]), __uint_as_float(o[2 * k + 1])),
                                   make_float2(inv_l, inv_l));
            pk[k] = row_has_keys ? pack2<FP16>(v.x, v.y) : 0u;
          }
          if (tma_out) {
            // columns 32q .. 32q+31: slab q / 2, 16-byte chunks 4 (q % 2) .. of the row, swizzled by row % 8
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int chunk = (q & 1) * 4 + k;
              *reinterpret_cast<uint4*>(qbuf + (q >> 1) * C::kSlabBytes + row * 128 + ((chunk ^ (row & 7)) << 4)) =
                  make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
            }
          } else if (row_valid && out_ok) {
            uint4* dst = reinterpret_cast<uint4*>(orow + q * 32);
#pragma unroll
            for (int k = 0; k < 4; ++k) dst[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
          }
        }
        if (tma_out) {
          fence_proxy_async_smem();
          mbar_arrive(bar(C::kBarOStaged + wg));
          if (quarter == 0 && lane == 0 && wait_bar(bar(C::kBarOStaged + wg), 0, wc) &&
              index_ok(q0 + (qt + 1) * kTile <= prm.total_q && h < prm.Hq)) {
            for (int hf = 0; hf < C::kHalves; ++hf)
              tma_store_3d(&tm_o, smem_u32(qbuf) + hf * C::kSlabBytes, hf * 64, h, q0 + qt * kTile);
            bulk_commit_group();
            bulk_wait_group_read0();  // the staging buffer must outlive the copy
          }
        }
        if (row_valid && out_ok) *lse_at = row_has_keys ? (m_used + lg2_approx(l_sum)) * kLn2 : -INFINITY;
      } else if (last < 0 && row_valid && out_ok) {
        // no key tile at all for this query tile
        uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
        for (int k = 0; k < D / 8; ++k) dst[k] = make_uint4(0u, 0u, 0u, 0u);
        *lse_at = -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Split-KV merge: for every (b, h, i), with the splits' partial results
// (O_s normalised by its own sum, LSE_s = log of that sum):
//   LSE = log sum_s exp(LSE_s),  O = sum_s exp(LSE_s - LSE) O_s,
// the same online-softmax rescaling as inside the kernel, applied once across
// splits (empty splits have LSE_s = -inf and weight 0; if every split is empty
// O = 0 and LSE = -inf). One warp per query row; D / 32 columns per lane.
template <int D, bool FP16>
__global__ void __launch_bounds__(128) fa_splitkv_combine_kernel(const float* __restrict__ part_o,
                                                                 const float* __restrict__ part_lse,
                                                                 uint16_t* __restrict__ out, float* __restrict__ lse,
                                                                 int n_splits, int BH, int Hq, int Nq) {
  const int lane = threadIdx.x % 32;
  const int64_t rowid = static_cast<int64_t>(blockIdx.x) * 4 + threadIdx.x / 32;  // (bh, i)
  const int64_t rows = static_cast<int64_t>(BH) * Nq;
  if (rowid >= rows) return;
  const int64_t stride = rows;  // between splits
  float mx = -INFINITY;
  for (int sp = lane; sp < n_splits; sp += 32) mx = fmaxf(mx, part_lse[sp * stride + rowid]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  const int bh = static_cast<int>(rowid / Nq), i = static_cast<int>(rowid % Nq);
  const int b = bh / Hq, h = bh % Hq;
  uint16_t* orow = out + ((static_cast<int64_t>(b) * Nq + i) * Hq + h) * D;
  constexpr int kPer = D / 32;  // columns per lane
  if (mx == -INFINITY) {
#pragma unroll
    for (int c = 0; c < kPer; ++c) orow[lane * kPer + c] = 0;
    if (lane == 0) lse[rowid] = -INFINITY;
    return;
  }
  float acc[kPer];
#pragma unroll
  for (int c = 0; c < kPer; ++c) acc[c] = 0.f;
  float wsum = 0.f;
  for (int sp = 0; sp < n_splits; ++sp) {
    const float w = ex2_approx((part_lse[sp * stride + rowid] - mx) * 1.44269504088896340736f);
    wsum += w;
    const float* src = part_o + (sp * stride + rowid) * D + lane * kPer;
#pragma unroll
    for (int c = 0; c < kPer; ++c) acc[c] = fmaf(w, src[c], acc[c]);
  }
  const float inv = 1.f / wsum;
#pragma unroll
  for (int c = 0; c < kPer; c += 2) {
    const uint32_t pk = pack2<FP16>(acc[c] * inv, acc[c + 1] * inv);
    *reinterpret_cast<uint32_t*>(orow + lane * kPer + c) = pk;
  }
  if (lane == 0) lse[rowid] = mx + lg2_approx(wsum) * kLn2;
}

}  // namespace fa
