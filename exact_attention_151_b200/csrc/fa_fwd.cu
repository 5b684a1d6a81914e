// fa_fwd.cu - fused exact-attention forward for B200 (sm_100a) and its C ABI.
//
// What one CTA computes: O and LSE for one 128-row query tile of one
// (batch, head), streaming over the visible 128-key tiles with an online
// softmax (running max and running sum per query row), so no N x N score or
// probability matrix ever reaches global memory:
//   * tiling Q / K / V and accumulating softmax numerator and denominator
//     block by block: llmtrend.com FlashAttention page, "how it works"
//     (split the sequence into blocks, accumulate attention in chunks);
//   * running max / running sum and rescaling the partial output: tuning
//     handbook ch. 3, "core idea" and the tiled routine in "engineering
//     implementation"; jsqmd.com page, tiling + streaming;
//   * one fused kernel for QK^T -> softmax -> PV: jsqmd.com page, kernel
//     fusion; prefetching the next K/V block while computing the current one:
//     mlqm.cn FA1/FA2 comparison, section 2.2;
//   * causal attention skips future positions: handbook ch. 3, practical notes.
//
// Blackwell mapping (not the Ampere design the pages sketch):
//   warp 5 (loader)   TMA 4-D tiled loads of Q once and K/V per key tile into a
//                     STAGES-deep ring of 128B-swizzled shared-memory tiles,
//                     completion tracked by mbarrier transaction counts;
//   warp 4 (MMA)      one thread issues tcgen05.mma: S_j = Q K_j^T into a
//                     double-buffered fp32 S in Tensor Memory, and
//                     O += P_j V_j with P_j read from Tensor Memory;
//   warps 0-3         one query row per thread (TMEM lane = row): load S_j,
//                     scale and mask, row max, exp2, row sum, write P_j as
//                     16-bit pairs over the first half of S_j's columns,
//                     rescale O when the row max grew, and finally normalise
//                     O by the row sum and write O and LSE.
// Since a TMEM lane holds a whole row, row max and row sum need no shuffles.
//
// Online-softmax bookkeeping (base 2, x = s * scale * log2(e)):
//   m is only raised when a tile's max exceeds it by more than
//   kRescaleThreshold; otherwise P = 2^(x - m) may reach 2^threshold, which
//   16-bit P and fp32 sums hold easily. O and l always share the same m, so
//   O / l and LSE = (m + log2 l) * ln 2 are exact up to rounding.

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cmath>
#include <mutex>

#include "fa.h"
#include "sm100.cuh"

namespace fa {

using namespace sm100;

// Device status word: bit 0 set when some wait ran out. Read and cleared by
// fa_status_sync. A static __device__ variable, so the library allocates nothing.
__device__ unsigned int g_status_word;

constexpr int kBM = 128;  // query rows per tile (= TMEM lanes)
constexpr int kBN = 128;  // keys per tile
constexpr int kThreads = 192;
constexpr int kMmaWarp = 4;
constexpr int kLoadWarp = 5;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr float kLn2 = 0.693147180559945309f;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 256;  // O accumulator columns [256, 256 + D)
constexpr uint32_t kMaxPolls = 1u << 28;
constexpr uint64_t kDefaultWaitLimitNs = 1ull << 30;  // about 1.07 s
constexpr uint64_t kDrainLimitNs = 20ull * 1000 * 1000;

template <int D>
struct Cfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kHalves = D / 64;                // 64-element (128 B) column slabs per row
  static constexpr int kSlabBytes = 128 * 128;          // one slab: 128 rows x 128 B
  static constexpr int kTileBytes = kHalves * kSlabBytes;
  static constexpr int kStages = (D == 128) ? 3 : 5;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kStages * kTileBytes;
  // barrier indices
  static constexpr int kBarQ = 0;
  static constexpr int kBarKFull = 1;
  static constexpr int kBarVFull = kBarKFull + kStages;
  static constexpr int kBarKVEmpty = kBarVFull + kStages;
  static constexpr int kBarSFull = kBarKVEmpty + kStages;  // [2]
  static constexpr int kBarPFull = kBarSFull + 2;          // [2]
  static constexpr int kBarODone = kBarPFull + 2;   // one phase per PV but the last
  static constexpr int kBarOFinal = kBarODone + 1;  // single phase: the last PV
  static constexpr int kBarDrain = kBarOFinal + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base slot, abort flag
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + slack to align the base to 1024 B
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Tile (query tile qt, key tile j) whose P is applied as P16 + (P - P16).
// Only the first key tile of the first query tile holds rows that see few
// keys (causal rows 0..127, or every row when N <= 128); there a single
// 16-bit rounding of P would weigh on the result about as much as the final
// rounding of O, so the residual is added with a second MMA pass. Elsewhere
// every row averages over more than 128 keys and the residual is negligible.
__device__ __forceinline__ bool split_p_tile(int qt, int j) { return qt == 0 && j == 0; }

struct WaitCtl {
  volatile int* abort;
  uint64_t limit_ns;
};

// Bounded wait for the phase of `bar` with `parity`. Returns false if this
// CTA is aborting or the wait ran out (which starts the abort and records
// the timeout in the status word).
__device__ __noinline__ bool wait_bar(uint32_t bar, uint32_t parity, WaitCtl w) {
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

// Short bounded wait used only while tearing down after an abort.
__device__ __noinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0; it < kMaxPolls; ++it) {
    if (mbar_try_wait(bar, parity)) return;
    if ((it & 15u) == 0 && globaltimer_ns() - t0 > kDrainLimitNs) return;
  }
}

// Warp-uniform wrapper: every lane polls, and the warp proceeds only if all did.
__device__ __forceinline__ bool warp_wait_bar(uint32_t bar, uint32_t parity, WaitCtl w) {
  const bool ok = wait_bar(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

template <int D, bool FP16>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, uint16_t* __restrict__ out, float* __restrict__ lse,
                  int N, int H, int n_tiles, float scale_log2, int causal, unsigned long long wait_limit_ns,
                  int withhold_v_load) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_smem = sbase + C::kQOff;
  auto k_smem = [&](int s) { return sbase + C::kKOff + s * C::kTileBytes; };
  auto v_smem = [&](int s) { return sbase + C::kVOff + s * C::kTileBytes; };
  auto bar = [&](int i) { return sbase + C::kBarOff + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  // Work item: CTAs of one (b, h) are adjacent (K/V reuse in L2); for causal
  // attention the heaviest query tiles of each head go first.
  const int bh = blockIdx.x / n_tiles;
  const int t = blockIdx.x % n_tiles;
  const int qt = causal ? (n_tiles - 1 - t) : t;
  const int b = bh / H;
  const int h = bh % H;
  const int n_kv = causal ? (qt + 1) : n_tiles;

  if (threadIdx.x == 0) {
    mbar_init(bar(C::kBarQ), 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar(C::kBarKFull + s), 1);
      mbar_init(bar(C::kBarVFull + s), 1);
      mbar_init(bar(C::kBarKVEmpty + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::kBarSFull + i), 1);
      mbar_init(bar(C::kBarPFull + i), 128);
    }
    mbar_init(bar(C::kBarODone), 1);
    mbar_init(bar(C::kBarOFinal), 1);
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
  const WaitCtl wc{abort_flag, wait_limit_ns};

  if (warp == kLoadWarp) {
    // ------------------------------------------------------------ loader
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int k_armed[C::kStages], v_armed[C::kStages];  // parity of the last arming, -1 if never
      for (int s = 0; s < C::kStages; ++s) k_armed[s] = v_armed[s] = -1;
      mbar_arrive_expect_tx(bar(C::kBarQ), C::kTileBytes);
      for (int hf = 0; hf < C::kHalves; ++hf)
        tma_load_4d(q_smem + hf * C::kSlabBytes, &tm_q, hf * 64, h, qt * kBM, b, bar(C::kBarQ));
      bool ok = true;
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % C::kStages;
        const uint32_t round = static_cast<uint32_t>(j / C::kStages);
        if (j >= C::kStages) {
          ok = wait_bar(bar(C::kBarKVEmpty + s), (round & 1u) ^ 1u, wc);
          if (!ok) break;
        }
        mbar_arrive_expect_tx(bar(C::kBarKFull + s), C::kTileBytes);
        for (int hf = 0; hf < C::kHalves; ++hf)
          tma_load_4d(k_smem(s) + hf * C::kSlabBytes, &tm_k, hf * 64, h, j * kBN, b, bar(C::kBarKFull + s));
        k_armed[s] = static_cast<int>(round & 1u);
        if (!(withhold_v_load && j == 0 && blockIdx.x == 0)) {
          mbar_arrive_expect_tx(bar(C::kBarVFull + s), C::kTileBytes);
          for (int hf = 0; hf < C::kHalves; ++hf)
            tma_load_4d(v_smem(s) + hf * C::kSlabBytes, &tm_v, hf * 64, h, j * kBN, b, bar(C::kBarVFull + s));
          v_armed[s] = static_cast<int>(round & 1u);
        }
      }
      // Let every load this thread issued land before shared memory is
      // released (immediate in a normal run, where all were consumed).
      (void)ok;
      drain_wait(bar(C::kBarQ), 0);
      for (int s = 0; s < C::kStages; ++s) {
        if (k_armed[s] >= 0) drain_wait(bar(C::kBarKFull + s), static_cast<uint32_t>(k_armed[s]));
        if (v_armed[s] >= 0) drain_wait(bar(C::kBarVFull + s), static_cast<uint32_t>(v_armed[s]));
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = instr_desc_f16(kBM, kBN, FP16, false);
      constexpr uint32_t idesc_pv = instr_desc_f16(kBM, D, FP16, true);
      bool ok = wait_bar(bar(C::kBarQ), 0, wc);
      for (int j = 0; ok && j <= n_kv; ++j) {
        if (j < n_kv) {
          // S_j = Q K_j^T  (K-major A and B, K = D in steps of 16)
          const int s = j % C::kStages;
          ok = wait_bar(bar(C::kBarKFull + s), static_cast<uint32_t>((j / C::kStages) & 1), wc);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem + static_cast<uint32_t>(j & 1) * kBN;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk / 4) * C::kSlabBytes + (kk % 4) * 32;
            const uint64_t a = smem_desc_sw128(q_smem + off, 16, 1024);
            const uint64_t bd = smem_desc_sw128(k_smem(s) + off, 16, 1024);
            mma_ss(d_tmem, a, bd, idesc_qk, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(C::kBarSFull + (j & 1)));
        }
        if (j >= 1) {
          // O += P_{j-1} V_{j-1}  (P from TMEM, V MN-major, K = 128 keys in steps of 16)
          const int jp = j - 1;
          const int sp = jp % C::kStages;
          ok = wait_bar(bar(C::kBarPFull + (jp & 1)), static_cast<uint32_t>((jp >> 1) & 1), wc);
          if (!ok) break;
          ok = wait_bar(bar(C::kBarVFull + sp), static_cast<uint32_t>((jp / C::kStages) & 1), wc);
          if (!ok) break;
          tc_fence_after();
          const uint32_t p_tmem = tmem + static_cast<uint32_t>(jp & 1) * kBN;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint64_t bd = smem_desc_sw128(v_smem(sp) + kk * 2048, C::kSlabBytes, 1024);
            mma_ts(tmem + kOCol, p_tmem + kk * 8, bd, idesc_pv, (jp > 0 || kk > 0) ? 1u : 0u);
          }
          if (split_p_tile(qt, jp)) {
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk) {
              const uint64_t bd = smem_desc_sw128(v_smem(sp) + kk * 2048, C::kSlabBytes, 1024);
              mma_ts(tmem + kOCol, p_tmem + 64 + kk * 8, bd, idesc_pv, 1u);
            }
          }
          // A parity wait is only unambiguous while the waiter is at most one
          // phase behind, which holds for the rescale waits on o_done (tile j
          // waits for PV_{j-1} after S_j, itself ordered after PV_{j-2}) but not
          // for the epilogue; the last PV therefore signals its own barrier.
          if (jp + 1 < n_kv) {
            mma_commit(bar(C::kBarODone));
          } else {
            mma_commit(bar(C::kBarOFinal));
          }
          if (jp + C::kStages < n_kv) mma_commit(bar(C::kBarKVEmpty + sp));
        }
      }
      if (!ok) {
        mma_commit(bar(C::kBarDrain));
        drain_wait(bar(C::kBarDrain), 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax / correction / epilogue
    const int row = warp * 32 + lane;
    const int qi = qt * kBM + row;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m_used = -INFINITY;
    float l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const uint32_t sbuf = static_cast<uint32_t>(j & 1) * kBN;
      ok = warp_wait_bar(bar(C::kBarSFull + (j & 1)), static_cast<uint32_t>((j >> 1) & 1), wc);
      if (!ok) break;
      tc_fence_after();
      float x[kBN];
      {
        uint32_t r[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tmem + lane_base + sbuf + c * 32, r[c]);
        tmem_wait_ld();
        const int kbase = j * kBN;
        const bool need_mask = (kbase + kBN > N) || (causal && j == qt);
        if (need_mask) {
          const int last = (causal ? min(N - 1, qi) : (N - 1)) - kbase;  // last visible column
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            x[c] = (c <= last) ? __uint_as_float(r[c / 32][c % 32]) * scale_log2 : -INFINITY;
        } else {
#pragma unroll
          for (int c = 0; c < kBN; ++c) x[c] = __uint_as_float(r[c / 32][c % 32]) * scale_log2;
        }
      }
      float mx0 = x[0], mx1 = x[1], mx2 = x[2], mx3 = x[3];
#pragma unroll
      for (int c = 4; c < kBN; c += 4) {
        mx0 = fmaxf(mx0, x[c]);
        mx1 = fmaxf(mx1, x[c + 1]);
        mx2 = fmaxf(mx2, x[c + 2]);
        mx3 = fmaxf(mx3, x[c + 3]);
      }
      const float m_tile = fmaxf(fmaxf(mx0, mx1), fmaxf(mx2, mx3));
      const float m_new = fmaxf(m_used, m_tile);
      float alpha = 1.f;
      const bool rescale = m_new > m_used + kRescaleThreshold;  // always true on the first tile
      if (rescale) {
        alpha = ex2_approx(m_used - m_new);  // 0 on the first tile (m_used = -inf)
        l_sum *= alpha;
        m_used = m_new;
      }
      float ls0 = 0.f, ls1 = 0.f, ls2 = 0.f, ls3 = 0.f;
      uint32_t pk[2][32];
#pragma unroll
      for (int c = 0; c < kBN; c += 4) {
        const float p0 = ex2_approx(x[c] - m_used);
        const float p1 = ex2_approx(x[c + 1] - m_used);
        const float p2 = ex2_approx(x[c + 2] - m_used);
        const float p3 = ex2_approx(x[c + 3] - m_used);
        ls0 += p0;
        ls1 += p1;
        ls2 += p2;
        ls3 += p3;
        pk[(c / 2) / 32][(c / 2) % 32] = pack2<FP16>(p0, p1);
        pk[(c / 2 + 1) / 32][(c / 2 + 1) % 32] = pack2<FP16>(p2, p3);
      }
      l_sum += (ls0 + ls1) + (ls2 + ls3);
      // P_j (16-bit pairs, key 2i in the low half of column i) over S_j's first 64 columns.
      tmem_st32(tmem + lane_base + sbuf, pk[0]);
      tmem_st32(tmem + lane_base + sbuf + 32, pk[1]);
      if (split_p_tile(qt, j)) {
        // Rows with only a few keys: also store the rounding residual P - P16
        // over the other 64 columns; the MMA adds it with a second pass.
        uint32_t lo[2][32];
#pragma unroll
        for (int c = 0; c < kBN; c += 2) {
          const float p0 = ex2_approx(x[c] - m_used);
          const float p1 = ex2_approx(x[c + 1] - m_used);
          const float2 hi = unpack2<FP16>(pk[(c / 2) / 32][(c / 2) % 32]);
          lo[(c / 2) / 32][(c / 2) % 32] = pack2<FP16>(p0 - hi.x, p1 - hi.y);
        }
        tmem_st32(tmem + lane_base + sbuf + 64, lo[0]);
        tmem_st32(tmem + lane_base + sbuf + 96, lo[1]);
      }
      tmem_wait_st();
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
        // O holds the sum up to tile j-1 under the old max: wait for PV_{j-1}, then scale.
        ok = warp_wait_bar(bar(C::kBarODone), static_cast<uint32_t>((j - 1) & 1), wc);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + kOCol + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tmem + lane_base + kOCol + c * 32, o);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar(C::kBarPFull + (j & 1)));
    }
    if (ok) ok = warp_wait_bar(bar(C::kBarOFinal), 0, wc);
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l_sum;
      const bool row_valid = qi < N;
      uint16_t* orow = out + ((static_cast<int64_t>(b) * N + qi) * H + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + kOCol + c * 32, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[i] = pack2<FP16>(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      if (row_valid) lse[(static_cast<int64_t>(b) * H + h) * N + qi] = (m_used + lg2_approx(l_sum)) * kLn2;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ====================================================================== host

namespace {

struct DeviceInfo {
  int checked = 0;  // 0 unknown, 1 ok, -1 unsupported
  unsigned configured = 0;  // bit per kernel instantiation: smem attribute set
};
constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool debug_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("FA_DEBUG");
    return e && *e && *e != '0';
  }();
  return on;
}

fa_status load_encoder() {
  static std::once_flag once;
  static fa_status st = FA_OK;
  std::call_once(once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    const cudaError_t e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) {
      st = FA_ERR_CUDA;
      cudaGetLastError();
    } else {
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  });
  return st;
}

// [B, N, H, D] 16-bit tensor viewed as 4-D (D, H, N, B), box (64, 1, 128, 1), 128B swizzle.
fa_status make_tmap(CUtensorMap* map, const void* base, int64_t B, int64_t N, int64_t H, int64_t D, bool fp16) {
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D * 2), static_cast<cuuint64_t>(H * D * 2),
                                 static_cast<cuuint64_t>(N * H * D * 2)};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = g_encode(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

fa_status check_device(int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
  *dev_out = dev;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceInfo& di = g_devices[dev];
  if (di.checked == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    di.checked = (major == 10 && minor == 0) ? 1 : -1;
  }
  return di.checked == 1 ? FA_OK : FA_ERR_UNSUPPORTED;
}

template <int D, bool FP16>
fa_status launch(int dev, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o, float* lse,
                 int64_t B, int64_t N, int64_t H, float scale, int causal, cudaStream_t stream, uint64_t limit_ns,
                 int withhold) {
  using C = Cfg<D>;
  auto kernel = fa_fwd_kernel<D, FP16>;
  const unsigned bit = 1u << ((D == 128 ? 2 : 0) + (FP16 ? 1 : 0));
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!(g_devices[dev].configured & bit)) {
      if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess) {
        cudaGetLastError();
        return FA_ERR_CUDA;
      }
      g_devices[dev].configured |= bit;
    }
  }
  const int64_t n_tiles = (N + kBM - 1) / kBM;
  const int64_t grid = n_tiles * B * H;
  const float scale_log2 = scale * 1.44269504088896340736f;
  kernel<<<static_cast<unsigned>(grid), kThreads, C::kSmemBytes, stream>>>(
      tq, tk, tv, static_cast<uint16_t*>(o), lse, static_cast<int>(N), static_cast<int>(H),
      static_cast<int>(n_tiles), scale_log2, causal ? 1 : 0, static_cast<unsigned long long>(limit_ns), withhold);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    if (debug_enabled()) std::fprintf(stderr, "[fa] launch failed: %s\n", cudaGetErrorString(e));
    return FA_ERR_CUDA;
  }
  if (debug_enabled()) {
    std::fprintf(stderr, "[fa] fwd D=%d %s B=%lld N=%lld H=%lld causal=%d grid=%lld smem=%d\n", D,
                 FP16 ? "fp16" : "bf16", (long long)B, (long long)N, (long long)H, causal, (long long)grid,
                 C::kSmemBytes);
  }
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t N, int64_t H,
                   int64_t D, float scale, int causal, fa_dtype dtype, fa_stream_t stream, uint64_t limit_ns,
                   int withhold) {
  if (B < 0 || N < 0 || H < 0) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || N == 0 || H == 0) return FA_OK;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) return FA_ERR_MISALIGNED;
  // int32 kernel indexing and TMA coordinate limits
  const int64_t n_tiles = (N + kBM - 1) / kBM;
  if (N > INT32_MAX || H > INT32_MAX || B > INT32_MAX) return FA_ERR_UNSUPPORTED;
  if (B * H > INT32_MAX / n_tiles) return FA_ERR_UNSUPPORTED;
  if (B * N > INT32_MAX / H) return FA_ERR_UNSUPPORTED;  // (b*N + i) * H + h fits int64 with room; keep rows int32
  if ((static_cast<double>(B) * N * H * D * 2) >= 1099511627776.0) return FA_ERR_UNSUPPORTED;  // < 2^40 B
  int dev = 0;
  fa_status st = check_device(&dev);
  if (st != FA_OK) return st;
  st = load_encoder();
  if (st != FA_OK) return st;
  const bool fp16 = dtype == FA_FP16;
  CUtensorMap tq, tk, tv;
  if (make_tmap(&tq, q, B, N, H, D, fp16) != FA_OK || make_tmap(&tk, k, B, N, H, D, fp16) != FA_OK ||
      make_tmap(&tv, v, B, N, H, D, fp16) != FA_OK)
    return FA_ERR_CUDA;
  if (limit_ns == 0) limit_ns = kDefaultWaitLimitNs;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (D == 128) {
    return fp16 ? launch<128, true>(dev, tq, tk, tv, o, lse, B, N, H, scale, causal, s, limit_ns, withhold)
                : launch<128, false>(dev, tq, tk, tv, o, lse, B, N, H, scale, causal, s, limit_ns, withhold);
  }
  return fp16 ? launch<64, true>(dev, tq, tk, tv, o, lse, B, N, H, scale, causal, s, limit_ns, withhold)
              : launch<64, false>(dev, tq, tk, tv, o, lse, B, N, H, scale, causal, s, limit_ns, withhold);
}

}  // namespace
}  // namespace fa

extern "C" {

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: null pointer, negative size, unknown dtype or non-finite scale";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: head dim not 64/128, size limit, or device is not sm_100";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED: a base pointer is not 16-byte aligned";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA runtime call failed";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a device-side wait ran out; outputs are invalid";
  }
  return "FA_ERR_UNKNOWN";
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t N, int64_t H,
                 int64_t D, float scale, int causal, fa_dtype dtype, fa_stream_t stream) {
  try {
    return fa::fwd_impl(q, k, v, o, lse, B, N, H, D, scale, causal, dtype, stream, 0, 0);
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

fa_status fa_fwd_debug(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t N,
                       int64_t H, int64_t D, float scale, int causal, fa_dtype dtype, fa_stream_t stream,
                       uint64_t wait_limit_ns, int withhold_v_load) {
  try {
    return fa::fwd_impl(q, k, v, o, lse, B, N, H, D, scale, causal, dtype, stream, wait_limit_ns,
                        withhold_v_load ? 1 : 0);
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

fa_status fa_status_sync(fa_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int word = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  if (cudaMemcpyFromSymbolAsync(&word, fa::g_status_word, sizeof(word), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_CUDA;
  }
  if (word != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbolAsync(fa::g_status_word, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    return FA_ERR_TIMEOUT;
  }
  return FA_OK;
}

}  // extern "C"
