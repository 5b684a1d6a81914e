// fa_bwd_kernel.cuh - backward of the fused attention for sm_100a.
//
// The backward recomputes the attention weights from Q, K and the forward's
// per-row log-sum-exp instead of storing them (the recomputation the jsqmd.com
// page describes: memory stays O(N)). With P_ij = exp(scale q_i.k_j - LSE_i)
// over the visible keys, D_i = dO_i . O_i and dS = P (dP - D):
//   dV = P^T dO,   dP = dO V^T,   dQ = scale dS K,   dK = scale dS^T Q.
//
// Three kernels, no atomics (deterministic):
//   fa_bwd_prep_kernel   D_i and LSE_i log2(e) into a workspace padded to
//                        whole 128-row tiles (pad rows: D = 0, LSE = +inf, so
//                        their weights are exactly 0);
//   fa_bwd_kernel<.., KV_SIDE = false>  one CTA per (128-query tile, b, h):
//                        S = Q K^T and dP = dO V^T into TMEM, dS = P (dP - D)
//                        by one thread per query row, dQ += dS K;
//   fa_bwd_kernel<.., KV_SIDE = true>   one CTA per (128-key tile, b, h):
//                        S^T = K Q^T and dP^T = V dO^T into TMEM, P^T and dS^T
//                        by one thread per key row, dV += P^T dO, dK += dS^T Q.
// Both share one warp-specialised skeleton: a TMA loader warp (the tile's two
// fixed operands once, the streamed pair into a two-stage ring), an MMA warp
// (converged, one elected lane issues tcgen05.mma), and four compute warps
// (TMEM lane = row). The operand of the accumulating MMAs that comes from the
// elementwise step (dS, P^T, dS^T) is written back to TMEM as 16-bit pairs
// over the first half of the score's columns, as P is in the forward.
#pragma once

#include <cuda.h>
#include <cstdint>

#include "fa_fwd_kernel.cuh"
#include "sm100.cuh"

namespace fa {
namespace bwd {

constexpr int kThreads = 192;
constexpr int kMma = 4;   // warp index
constexpr int kLoad = 5;  // warp index

template <int D>
struct Cfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kSlabBytes = 128 * 128;
  static constexpr int kTileBytes = kHalves * kSlabBytes;
  static constexpr int kStages = 2;
  static constexpr int kXOff = 0;                              // fixed operands X1, X2
  static constexpr int kYOff = kXOff + 2 * kTileBytes;          // ring of (Y1, Y2) pairs
  static constexpr int kBarOff = kYOff + kStages * 2 * kTileBytes;
  static constexpr int kBarX = 0;
  static constexpr int kBarYFull = 1;                 // [kStages]
  static constexpr int kBarYEmpty = 1 + kStages;      // [kStages]
  static constexpr int kBarSFull = 1 + 2 * kStages;   // scores ready
  static constexpr int kBarPFull = kBarSFull + 1;     // elementwise results written (128 arrivals)
  static constexpr int kBarDone = kBarPFull + 1;      // last accumulating MMA finished
  static constexpr int kBarDrain = kBarDone + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kWsOff = kBarOff + 128;    // per compute warp 2 x 128 floats (key side)
  static constexpr int kMiscOff = kWsOff + 4 * 1024;
  static_assert(kNumBars * 8 <= 128, "barrier area");
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  // TMEM columns: score A (S or S^T), score B (dP or dP^T), accumulators
  static constexpr uint32_t kColSA = 0, kColSB = 128, kColAcc0 = 256, kColAcc1 = 256 + D;
};

struct Params {
  const float* ws_d;    // [B*H, Npad]: D_i = dO_i . O_i (0 on pad rows)
  const float* ws_l;    // [B*H, Npad]: LSE_i * log2(e) (+inf on pad rows)
  uint16_t* out0;       // query side: dQ;   key side: dK
  uint16_t* out1;       // key side: dV
  int N, H, Npad, n_tiles;
  float scale_log2;     // scale * log2(e)
  float scale;
  int causal;
  unsigned long long wait_limit_ns;
};

// D_i and LSE_i log2(e) per row, padded to whole tiles. One warp per row.
template <int D, bool FP16>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const uint16_t* __restrict__ o,
                                                          const uint16_t* __restrict__ dout,
                                                          const float* __restrict__ lse, float* __restrict__ ws_d,
                                                          float* __restrict__ ws_l, int BH, int N, int H, int Npad) {
  const int lane = threadIdx.x % 32;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + threadIdx.x / 32;  // (bh, i) over the padded rows
  if (r >= static_cast<int64_t>(BH) * Npad) return;
  const int bh = static_cast<int>(r / Npad), i = static_cast<int>(r % Npad);
  if (i >= N) {
    if (lane == 0) {
      ws_d[r] = 0.f;
      ws_l[r] = INFINITY;
    }
    return;
  }
  const int b = bh / H, h = bh % H;
  const int64_t base = ((static_cast<int64_t>(b) * N + i) * H + h) * D;
  constexpr int kPer = D / 32;  // elements per lane (2 or 4)
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < kPer; c += 2) {
    const float2 x = unpack2<FP16>(*reinterpret_cast<const uint32_t*>(o + base + lane * kPer + c));
    const float2 y = unpack2<FP16>(*reinterpret_cast<const uint32_t*>(dout + base + lane * kPer + c));
    acc = fmaf(x.x, y.x, fmaf(x.y, y.y, acc));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    ws_d[r] = acc;
    ws_l[r] = lse[static_cast<int64_t>(bh) * N + i] * 1.44269504088896340736f;
  }
}

// KV_SIDE = false: tile of 128 queries; X1 = Q, X2 = dO fixed, stream (K_t, V_t)
//   over key tiles t = 0 .. last; out0 = dQ.
// KV_SIDE = true:  tile of 128 keys; X1 = K, X2 = V fixed, stream (Q_t, dO_t)
//   over query tiles t = first .. n_tiles-1; out0 = dK, out1 = dV.
template <int D, bool FP16, bool KV_SIDE>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_x1, const __grid_constant__ CUtensorMap tm_x2,
                  const __grid_constant__ CUtensorMap tm_y1, const __grid_constant__ CUtensorMap tm_y2,
                  const Params prm) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  auto x_smem = [&](int i) { return sbase + C::kXOff + i * C::kTileBytes; };
  auto y_smem = [&](int s, int i) { return sbase + C::kYOff + (2 * s + i) * C::kTileBytes; };
  auto bar = [&](int i) { return sbase + C::kBarOff + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int N = prm.N;
  const int causal = prm.causal;
  const int tile = static_cast<int>(blockIdx.x) % prm.n_tiles;  // this CTA's query (or key) tile
  const int bh = static_cast<int>(blockIdx.x) / prm.n_tiles;
  const int b = bh / prm.H, h = bh % prm.H;
  // streamed tiles: query side: keys 0 .. (causal ? tile : n_tiles-1);
  //                 key side:   queries (causal ? tile : 0) .. n_tiles-1
  const int t_first = KV_SIDE ? (causal ? tile : 0) : 0;
  const int t_last = KV_SIDE ? prm.n_tiles - 1 : (causal ? tile : prm.n_tiles - 1);
  const int n_t = t_last - t_first + 1;

  if (threadIdx.x == 0) {
    mbar_init(bar(C::kBarX), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(C::kBarYFull + s), 1);
      mbar_init(bar(C::kBarYEmpty + s), 1);
    }
    mbar_init(bar(C::kBarSFull), 1);
    mbar_init(bar(C::kBarPFull), 128);
    mbar_init(bar(C::kBarDone), 1);
    mbar_init(bar(C::kBarDrain), 1);
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
  const int row0 = b * N;  // first row of this (b) in the [B*N, H, D] views

  if (warp == kLoad) {
    // ------------------------------------------------------------ loader (converged warp)
    if (lane == 0) {
      tma_prefetch_desc(&tm_x1);
      tma_prefetch_desc(&tm_x2);
      tma_prefetch_desc(&tm_y1);
      tma_prefetch_desc(&tm_y2);
    }
    __syncwarp();
    mbar_arrive_expect_tx_elect(bar(C::kBarX), 2 * C::kTileBytes);
    for (int hf = 0; hf < C::kHalves; ++hf) {
      tma_load_3d_elect(x_smem(0) + hf * C::kSlabBytes, &tm_x1, hf * 64, h, row0 + tile * kTile, bar(C::kBarX));
      tma_load_3d_elect(x_smem(1) + hf * C::kSlabBytes, &tm_x2, hf * 64, h, row0 + tile * kTile, bar(C::kBarX));
    }
    int issued = 0;
    for (int t = 0; t < n_t; ++t) {
      const int s = t % C::kStages;
      if (t >= C::kStages &&
          !warp_wait_bar(bar(C::kBarYEmpty + s), static_cast<uint32_t>(((t / C::kStages) & 1) ^ 1), wc))
        break;
      const int row = row0 + (t_first + t) * kTile;
      mbar_arrive_expect_tx_elect(bar(C::kBarYFull + s), 2 * C::kTileBytes);
      for (int hf = 0; hf < C::kHalves; ++hf) {
        tma_load_3d_elect(y_smem(s, 0) + hf * C::kSlabBytes, &tm_y1, hf * 64, h, row, bar(C::kBarYFull + s));
        tma_load_3d_elect(y_smem(s, 1) + hf * C::kSlabBytes, &tm_y2, hf * 64, h, row, bar(C::kBarYFull + s));
      }
      issued = t + 1;
    }
    // let the copies this warp issued land before shared memory is released
    drain_wait(bar(C::kBarX), 0);
    for (int s = 0; s < C::kStages && s < issued; ++s) {
      const int tl = s + ((issued - 1 - s) / C::kStages) * C::kStages;
      drain_wait(bar(C::kBarYFull + s), static_cast<uint32_t>((tl / C::kStages) & 1));
    }
  } else if (warp == kMma) {
    // ------------------------------------------------------------ MMA issue (converged warp)
    constexpr uint32_t idesc_score = instr_desc_f16(kTile, kTile, FP16, false);
    constexpr uint32_t idesc_acc = instr_desc_f16(kTile, D, FP16, true);
    constexpr uint64_t kTileStep = C::kTileBytes >> 4;
    const uint64_t x_desc0 = smem_desc_sw128(x_smem(0), 16, 1024);  // K-major views
    const uint64_t y_desc0 = smem_desc_sw128(y_smem(0, 0), 16, 1024);
    const uint64_t y_mn0 = smem_desc_sw128(y_smem(0, 0), C::kSlabBytes, 1024);  // MN-major view of the same tiles
    bool ok = warp_wait_bar(bar(C::kBarX), 0, wc);
    for (int t = 0; ok && t < n_t; ++t) {
      const int s = t % C::kStages;
      ok = warp_wait_bar(bar(C::kBarYFull + s), static_cast<uint32_t>((t / C::kStages) & 1), wc);
      if (!ok) break;
      tc_fence_after();
      // score A = X1 Y1^T (S or S^T), score B = X2 Y2^T (dP or dP^T); K = D in steps of 16
      const uint64_t y1 = y_desc0 + static_cast<uint64_t>(2 * s) * kTileStep;
      const uint64_t y2 = y1 + kTileStep;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>(((kk / 4) * C::kSlabBytes + (kk % 4) * 32) >> 4);
        mma_ss_elect(tmem + C::kColSA, x_desc0 + off, y1 + off, idesc_score, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>(((kk / 4) * C::kSlabBytes + (kk % 4) * 32) >> 4);
        mma_ss_elect(tmem + C::kColSB, x_desc0 + kTileStep + off, y2 + off, idesc_score, kk > 0 ? 1u : 0u);
      }
      mma_commit_elect(bar(C::kBarSFull));
      ok = warp_wait_bar(bar(C::kBarPFull), static_cast<uint32_t>(t & 1), wc);
      if (!ok) break;
      tc_fence_after();
      // accumulate: K = 128 rows of the streamed tiles in steps of 16 (B operand MN-major)
      const uint64_t y1mn = y_mn0 + static_cast<uint64_t>(2 * s) * kTileStep;
      const uint64_t y2mn = y1mn + kTileStep;
#pragma unroll
      for (int kk = 0; kk < kTile / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>(kk * (2048 >> 4));
        const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
        if constexpr (KV_SIDE) {
          mma_ts_elect(tmem + C::kColAcc1, tmem + C::kColSA + kk * 8, y2mn + off, idesc_acc, acc);  // dV += P^T dO
          mma_ts_elect(tmem + C::kColAcc0, tmem + C::kColSB + kk * 8, y1mn + off, idesc_acc, acc);  // dK += dS^T Q
        } else {
          mma_ts_elect(tmem + C::kColAcc0, tmem + C::kColSA + kk * 8, y1mn + off, idesc_acc, acc);  // dQ += dS K
        }
      }
      if (t + C::kStages < n_t) mma_commit_elect(bar(C::kBarYEmpty + s));
      if (t == n_t - 1) mma_commit_elect(bar(C::kBarDone));
    }
    if (!ok) {
      mma_commit_elect(bar(C::kBarDrain));
      drain_wait(bar(C::kBarDrain), 0);
    }
  } else {
    // ------------------------------------------------------------ compute warps (TMEM lane = row)
    const int row = warp * 32 + lane;
    const int r_abs = tile * kTile + row;  // this thread's query (or key) index
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const float c = prm.scale_log2;
    const float* ws_d = prm.ws_d + static_cast<int64_t>(bh) * prm.Npad;
    const float* ws_l = prm.ws_l + static_cast<int64_t>(bh) * prm.Npad;
    float row_d = 0.f, row_l = 0.f;
    if constexpr (!KV_SIDE) {
      row_d = ws_d[r_abs];
      row_l = ws_l[r_abs];
    }
    // key side: each warp keeps its own copy of the current query tile's
    // LSE log2(e) and D values (warp-local, so no barrier across warps)
    float* ws_s_l = reinterpret_cast<float*>(smem + C::kWsOff) + warp * 2 * kTile;
    float* ws_s_d = ws_s_l + kTile;
    bool ok = true;
    for (int t = 0; t < n_t; ++t) {
      const int cbase = (t_first + t) * kTile;  // first column index (key, or query) of this tile
      if constexpr (KV_SIDE) {
        __syncwarp();  // every lane is done with the previous tile's values
#pragma unroll
        for (int i = 0; i < kTile / 32; ++i) {
          ws_s_l[i * 32 + lane] = ws_l[cbase + i * 32 + lane];
          ws_s_d[i * 32 + lane] = ws_d[cbase + i * 32 + lane];
        }
        __syncwarp();
      }
      ok = warp_wait_bar(bar(C::kBarSFull), static_cast<uint32_t>(t & 1), wc);
      if (!ok) break;
      tc_fence_after();
      // Columns in chunks of 32: the 16-bit results of chunk ch go to packed
      // columns 16 ch .. 16 ch + 15, which only hold scores already read.
      const bool masked = KV_SIDE ? (causal && cbase == tile * kTile)
                                  : (cbase + kTile > N || (causal && cbase == tile * kTile));
#pragma unroll
      for (int ch = 0; ch < kTile / 32; ++ch) {
        uint32_t sa[32], sb[32];
        tmem_ld32(tmem + lane_base + C::kColSA + ch * 32, sa);
        tmem_ld32(tmem + lane_base + C::kColSB + ch * 32, sb);
        tmem_wait_ld();
        uint32_t pk_a[16], pk_b[16];  // query side: dS (pk_a); key side: P^T (pk_a), dS^T (pk_b)
#pragma unroll
        for (int q = 0; q < 32; q += 2) {
          float p[2], ds[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float sv = __uint_as_float(sa[q + e]);
            const float dpv = __uint_as_float(sb[q + e]);
            const int cidx = cbase + ch * 32 + q + e;
            if constexpr (KV_SIDE) {
              // row = key r_abs, column = query cidx; pad queries have LSE = +inf, so P = 0
              const bool vis = !masked || cidx >= r_abs;
              p[e] = vis ? ex2_approx(fmaf(sv, c, -ws_s_l[ch * 32 + q + e])) : 0.f;
              ds[e] = p[e] * (dpv - ws_s_d[ch * 32 + q + e]);
            } else {
              // row = query r_abs, column = key cidx
              const bool vis = !masked || (cidx < N && (!causal || cidx <= r_abs));
              p[e] = vis ? ex2_approx(fmaf(sv, c, -row_l)) : 0.f;
              ds[e] = p[e] * (dpv - row_d);
            }
          }
          if constexpr (KV_SIDE) {
            pk_a[q / 2] = pack2<FP16>(p[0], p[1]);
            pk_b[q / 2] = pack2<FP16>(ds[0], ds[1]);
          } else {
            pk_a[q / 2] = pack2<FP16>(ds[0], ds[1]);
          }
        }
        tmem_st16(tmem + lane_base + C::kColSA + ch * 16, pk_a);
        if constexpr (KV_SIDE) tmem_st16(tmem + lane_base + C::kColSB + ch * 16, pk_b);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(C::kBarPFull));
    }
    if (ok) ok = warp_wait_bar(bar(C::kBarDone), 0, wc);
    if (ok) {
      tc_fence_after();
      const bool row_valid = r_abs < N;
      const int64_t obase = ((static_cast<int64_t>(b) * N + r_abs) * prm.H + h) * D;
#pragma unroll
      for (int which = 0; which < (KV_SIDE ? 2 : 1); ++which) {
        // query side: dQ (scaled); key side: which 0 = dK (scaled, acc0), 1 = dV (acc1)
        const uint32_t col = which == 0 ? C::kColAcc0 : C::kColAcc1;
        const float mul = which == 0 ? prm.scale : 1.f;
        uint16_t* dst_row = (which == 0 ? prm.out0 : prm.out1) + obase;
#pragma unroll
        for (int q = 0; q < D / 32; ++q) {
          uint32_t a[32];
          tmem_ld32(tmem + lane_base + col + q * 32, a);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k)
            pk[k] = pack2<FP16>(__uint_as_float(a[2 * k]) * mul, __uint_as_float(a[2 * k + 1]) * mul);
          if (row_valid) {
            uint4* dst = reinterpret_cast<uint4*>(dst_row + q * 32);
#pragma unroll
            for (int k = 0; k < 4; ++k) dst[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
          }
        }
      }
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
