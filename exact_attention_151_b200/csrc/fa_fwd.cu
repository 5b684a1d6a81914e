// fa_fwd.cu - host side of the fused exact attention: argument checks, TMA
// tensor-map encoding, launches, and the C ABI declared in fa.h. The forward
// kernel is in fa_fwd_kernel.cuh, the backward kernels in fa_bwd_kernel.cuh
// (one translation unit, so every kernel reports into one status word).

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cfloat>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <mutex>

#include "fa.h"
#include "fa_bwd_kernel.cuh"
#include "fa_fwd_kernel.cuh"

namespace fa {

namespace {

constexpr uint64_t kDefaultWaitLimitNs = 1ull << 30;  // about 1.07 s

thread_local char g_last_error[256] = "";

void set_error(const char* where, cudaError_t e) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%d)", where, cudaGetErrorString(e), static_cast<int>(e));
}

struct DeviceInfo {
  int checked = 0;  // 0 unknown, 1 ok, -1 unsupported
  unsigned configured = 0;  // bit per kernel instantiation: smem attribute set (layout at each launch)
};
constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// FA_DEBUG, or the pages' names for their library's debug switch
// (FLASH_ATTN_DEBUG, FLASH_ATTENTION_DEBUG), read once.
bool debug_enabled() {
  static const bool on = [] {
    for (const char* name : {"FA_DEBUG", "FLASH_ATTN_DEBUG", "FLASH_ATTENTION_DEBUG"}) {
      const char* e = std::getenv(name);
      if (e && *e && *e != '0') return true;
    }
    return false;
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
      set_error("cudaGetDriverEntryPointByVersion(cuTensorMapEncodeTiled)", e);
      cudaGetLastError();
    } else {
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  });
  return st;
}

// A [rows, H, D] 16-bit tensor (a dense [B, N, H, D] tensor is B*N rows)
// viewed as 3-D (D, H, rows), box (64, box_h, box_rows) (default one head by
// 128 rows), 128B swizzle; rows past the end are zero-filled by TMA.
fa_status make_tmap(CUtensorMap* map, const void* base, int64_t rows, int64_t H, int64_t D, bool fp16,
                    uint32_t box_h = 1, uint32_t box_rows = 128) {
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D * 2), static_cast<cuuint64_t>(H * D * 2)};
  const cuuint32_t box[3] = {64, box_h, box_rows};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

fa_status check_device(int* dev_out) {
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    set_error("cudaGetDevice", e);
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

// Problem shape as the host sees it (dense when cu_q == nullptr).
struct Shape {
  const int* cu_q;
  const int* cu_k;
  int64_t B, Nq, Nk, total_q, total_k, max_nq, Hq, Hkv, D;
  int pack_g = 0;         // packed heads (dense, Nq * G <= 128): G = Hq / Hkv, else 0
  int n_splits = 1;       // split-KV (dense shapes): number of key ranges
  int split_tiles = 0;    // key tiles per range
  float* part_o = nullptr;
  float* part_lse = nullptr;
};

template <int D, bool FP16>
fa_status launch(int dev, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& to,
                 void* o, float* lse,
                 const Shape& sh, float scale, int causal, cudaStream_t stream, uint64_t limit_ns, int withhold) {
  using C = Cfg<D>;
  // packed heads leave the second query tile free: it takes a second key range
  const bool pair = sh.pack_g && sh.n_splits > 1;
  auto kernel = pair ? fa_fwd_kernel<D, FP16, true> : fa_fwd_kernel<D, FP16, false>;
  // configured bits: 0-3 unpaired forward, 4-11 backward, 12-15 paired forward
  const unsigned bit = 1u << ((pair ? 12 : 0) + (D == 128 ? 2 : 0) + (FP16 ? 1 : 0));
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!(g_devices[dev].configured & bit)) {
      // The kernel moves registers between warpgroups (setmaxnreg); that is only
      // safe if the launch gives every thread exactly the count the split was
      // sized for. Refuse to launch otherwise (an increase would never return).
      cudaFuncAttributes attr;
      cudaError_t e = cudaFuncGetAttributes(&attr, kernel);
      if (e != cudaSuccess) {
        set_error("cudaFuncGetAttributes", e);
        cudaGetLastError();
        return FA_ERR_CUDA;
      }
      if (attr.numRegs != static_cast<int>(kLaunchRegs)) {
        std::snprintf(g_last_error, sizeof(g_last_error),
                      "kernel built with %d registers per thread, register split expects %u", attr.numRegs,
                      kLaunchRegs);
        return FA_ERR_UNSUPPORTED;
      }
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
      if (e != cudaSuccess) {
        set_error("cudaFuncSetAttribute", e);
        cudaGetLastError();
        return FA_ERR_CUDA;
      }
      g_devices[dev].configured |= bit;
    }
  }
  Params prm;
  prm.out = static_cast<uint16_t*>(o);
  prm.lse = lse;
  prm.cu_q = sh.cu_q;
  prm.cu_k = sh.cu_k;
  prm.Nq = static_cast<int>(sh.Nq);
  prm.Nk = static_cast<int>(sh.Nk);
  prm.total_q = static_cast<int>(sh.total_q);
  prm.total_k = static_cast<int>(sh.total_k);
  prm.Hq = static_cast<int>(sh.Hq);
  prm.Hkv = static_cast<int>(sh.Hkv);
  prm.BH = static_cast<int>(sh.pack_g ? sh.B * sh.Hkv : sh.B * sh.Hq);
  prm.BHq = static_cast<int>(sh.B * sh.Hq);
  prm.pack_g = sh.pack_g;
  prm.max_nq = static_cast<int>(sh.max_nq);
  prm.n_blocks = sh.pack_g ? 1 : static_cast<int>((sh.max_nq + kBlockRows - 1) / kBlockRows);
  // Softmax runs in base 2: x = s * scale * log2(e). A zero (or subnormal)
  // factor is replaced by +-FLT_MIN: every weight then still rounds to
  // exactly 1 (|s| < 2^40 for 16-bit inputs) while masked keys keep weight 0.
  float c = scale * 1.44269504088896340736f;
  if (std::fabs(c) < FLT_MIN) c = std::signbit(c) ? -FLT_MIN : FLT_MIN;
  prm.scale_log2 = c;
  prm.causal = causal ? 1 : 0;
  prm.wait_limit_ns = static_cast<unsigned long long>(limit_ns);
  prm.withhold_v_load = withhold;
  prm.n_splits = sh.n_splits;
  prm.split_tiles = sh.split_tiles;
  prm.part_o = sh.part_o;
  prm.part_lse = sh.part_lse;
  const int64_t cta_splits = pair ? (sh.n_splits + 1) / 2 : sh.n_splits;
  const int64_t grid = static_cast<int64_t>(prm.n_blocks) * prm.BH * cta_splits;
  kernel<<<static_cast<unsigned>(grid), kThreads, C::kSmemBytes, stream>>>(tq, tk, tv, to, prm);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error("kernel launch", e);
    if (debug_enabled()) std::fprintf(stderr, "[fa] launch failed: %s\n", cudaGetErrorString(e));
    return FA_ERR_CUDA;
  }
  if (sh.n_splits > 1) {
    const int64_t rows = sh.B * sh.Hq * sh.Nq;
    fa_splitkv_combine_kernel<D, FP16><<<static_cast<unsigned>((rows + 3) / 4), 128, 0, stream>>>(
        sh.part_o, sh.part_lse, static_cast<uint16_t*>(o), lse, sh.n_splits, static_cast<int>(sh.B * sh.Hq),
        static_cast<int>(sh.Hq), static_cast<int>(sh.Nq));
    const cudaError_t e2 = cudaGetLastError();
    if (e2 != cudaSuccess) {
      set_error("combine launch", e2);
      return FA_ERR_CUDA;
    }
  }
  if (debug_enabled()) {
    std::fprintf(stderr, "[fa] fwd D=%d %s B=%lld Nq=%lld Nk=%lld Hq=%lld Hkv=%lld %s causal=%d splits=%d%s grid=%lld smem=%d\n",
                 D, FP16 ? "fp16" : "bf16", (long long)sh.B, (long long)sh.Nq, (long long)sh.Nk, (long long)sh.Hq,
                 (long long)sh.Hkv, sh.cu_q ? "packed" : "dense", causal, sh.n_splits, pair ? " paired" : "",
                 (long long)grid, C::kSmemBytes);
  }
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxSplits = 64;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace of a split-KV call: fp32 partial O [n_splits, B*Hq, Nq, D], then
// fp32 partial LSE [n_splits, B*Hq, Nq], each 256-byte aligned.
size_t splitkv_bytes(int64_t n_splits, int64_t BH, int64_t Nq, int64_t D) {
  return align256(static_cast<size_t>(n_splits * BH * Nq * D) * 4) + align256(static_cast<size_t>(n_splits * BH * Nq) * 4);
}

// Packed heads (one query tile per key/value head holds all G = Hq / Hkv query
// heads for every query position) for dense shapes with Nq * G <= 128, G > 1.
int64_t pack_group(int64_t Nq, int64_t Hq, int64_t Hkv) {
  if (Hkv < 1 || Hq % Hkv != 0) return 0;
  const int64_t g = Hq / Hkv;
  return (g > 1 && Nq >= 1 && Nq * g <= kTile) ? g : 0;
}

// Number of key ranges: when the query side alone fills less than half the
// SMs, as many ranges as keep the CTAs within one wave (one CTA per SM; with
// packed heads a CTA takes two ranges, one per query tile), never more than the
// key tiles or kMaxSplits; the count is then evened so every range has the same
// number of tiles.
int resolve_splits(int requested, int64_t B, int64_t Nq, int64_t Nk, int64_t Hq, int64_t Hkv, int sm_count,
                   int* tiles_out) {
  const int64_t n_kt = (Nk + kTile - 1) / kTile;
  const bool packed = pack_group(Nq, Hq, Hkv) != 0;
  const int64_t base = packed ? B * Hkv : ((Nq + kBlockRows - 1) / kBlockRows) * B * Hq;
  int64_t want = requested;
  if (want <= 0) want = (base >= sm_count / 2 || n_kt < 2) ? 1 : (packed ? 2 : 1) * (sm_count / base);
  want = std::max<int64_t>(1, std::min<int64_t>({want, n_kt > 0 ? n_kt : 1, kMaxSplits}));
  const int64_t tiles = (n_kt + want - 1) / want;
  const int64_t splits = tiles > 0 ? (n_kt + tiles - 1) / tiles : 1;
  *tiles_out = static_cast<int>(tiles);
  return static_cast<int>(std::max<int64_t>(1, splits));
}

int device_sm_count(int dev) {
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

fa_status fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, const Shape& sh, float scale,
                   int causal, fa_dtype dtype, fa_stream_t stream, uint64_t limit_ns, int withhold) {
  if (sh.B < 0 || sh.Nq < 0 || sh.Nk < 0 || sh.Hq < 0 || sh.Hkv < 0 || sh.total_q < 0 || sh.total_k < 0 ||
      sh.max_nq < 0)
    return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (sh.Hq > 0 && (sh.Hkv < 1 || sh.Hq % sh.Hkv != 0)) return FA_ERR_INVALID_ARG;
  if (sh.D != 64 && sh.D != 128) return FA_ERR_UNSUPPORTED;
  if (sh.B == 0 || sh.Hq == 0 || sh.total_q == 0 || sh.max_nq == 0) return FA_OK;
  if (!q || !o || !lse || (sh.total_k > 0 && (!k || !v))) return FA_ERR_INVALID_ARG;
  if (sh.cu_q && !sh.cu_k) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(o) || !aligned16(lse) || (sh.total_k > 0 && (!aligned16(k) || !aligned16(v))))
    return FA_ERR_MISALIGNED;
  // int32 kernel indexing, TMA coordinate and tensor-size limits
  const int64_t n_blocks = (sh.max_nq + kBlockRows - 1) / kBlockRows;
  if (sh.total_q > INT32_MAX - 2 * kBlockRows || sh.total_k > INT32_MAX - 2 * kBlockRows || sh.Hq > INT32_MAX ||
      sh.B > INT32_MAX || sh.max_nq > INT32_MAX - 2 * kBlockRows)
    return FA_ERR_UNSUPPORTED;
  if (sh.B * sh.Hq > INT32_MAX / n_blocks) return FA_ERR_UNSUPPORTED;
  if (static_cast<double>(sh.total_q) * sh.Hq * sh.D * 2 >= 1099511627776.0 ||
      static_cast<double>(sh.total_k) * sh.Hkv * sh.D * 2 >= 1099511627776.0)
    return FA_ERR_UNSUPPORTED;  // each tensor < 2^40 bytes
  int dev = 0;
  fa_status st = check_device(&dev);
  if (st != FA_OK) return st;
  st = load_encoder();
  if (st != FA_OK) return st;
  const bool fp16 = dtype == FA_FP16;
  // With no keys at all nothing is ever loaded from K or V; the maps only need
  // a valid, aligned base.
  const void* kb = sh.total_k > 0 ? k : q;
  const void* vb = sh.total_k > 0 ? v : q;
  const int64_t krows = sh.total_k > 0 ? sh.total_k : 1;
  const int64_t khead = sh.total_k > 0 ? sh.Hkv : 1;
  CUtensorMap tq, tk, tv, to;
  Shape shp = sh;
  shp.pack_g = sh.cu_q == nullptr ? static_cast<int>(pack_group(sh.Nq, sh.Hq, sh.Hkv)) : 0;
  const fa_status mq = shp.pack_g ? make_tmap(&tq, q, sh.total_q, sh.Hq, sh.D, fp16, static_cast<uint32_t>(shp.pack_g),
                                              static_cast<uint32_t>(sh.Nq))
                                  : make_tmap(&tq, q, sh.total_q, sh.Hq, sh.D, fp16);
  if (mq != FA_OK || make_tmap(&tk, kb, krows, khead, sh.D, fp16) != FA_OK ||
      make_tmap(&tv, vb, krows, khead, sh.D, fp16) != FA_OK || make_tmap(&to, o, sh.total_q, sh.Hq, sh.D, fp16) != FA_OK)
    return FA_ERR_CUDA;
  if (limit_ns == 0) limit_ns = kDefaultWaitLimitNs;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (sh.D == 128) {
    return fp16 ? launch<128, true>(dev, tq, tk, tv, to, o, lse, shp, scale, causal, s, limit_ns, withhold)
                : launch<128, false>(dev, tq, tk, tv, to, o, lse, shp, scale, causal, s, limit_ns, withhold);
  }
  return fp16 ? launch<64, true>(dev, tq, tk, tv, to, o, lse, shp, scale, causal, s, limit_ns, withhold)
              : launch<64, false>(dev, tq, tk, tv, to, o, lse, shp, scale, causal, s, limit_ns, withhold);
}

Shape dense_shape(int64_t B, int64_t Nq, int64_t Nk, int64_t Hq, int64_t Hkv, int64_t D) {
  Shape sh{nullptr, nullptr, B, Nq, Nk, B * Nq, B * Nk, Nq, Hq, Hkv, D};
  if (B < 0 || Nq < 0 || Nk < 0) sh.B = -1;  // rejected by fwd_impl
  return sh;
}

// ---------------------------------------------------------------- backward

// Workspace of the backward: D_i = dO_i . O_i, then LSE_i log2(e), each fp32
// [B*Hq, Npad] with Npad = Nq rounded up to whole 128-row tiles, 256-byte aligned.
// -D and -LSE log2(e) per padded row, then the two gradient kernels' work-item counters
size_t bwd_ws_bytes(int64_t B, int64_t Nq, int64_t Hq) {
  if (B <= 0 || Hq <= 0) return 0;  // nothing to do
  const int64_t npad = (Nq + kTile - 1) / kTile * kTile;
  return 2 * align256(static_cast<size_t>(B * Hq * npad) * 4) + 256;
}

template <int D, bool FP16, bool KV_SIDE>
fa_status bwd_launch(int dev, const CUtensorMap& x1, const CUtensorMap& x2, const CUtensorMap& y1,
                     const CUtensorMap& y2, const bwd::Params& prm, int64_t grid, cudaStream_t stream) {
  constexpr int kSmem = KV_SIDE ? bwd::Cfg<D>::kSmemBytes : bwd::CfgQ<D>::kSmemBytes;
  auto kernel = KV_SIDE ? bwd::fa_bwd_dkdv_kernel<D, FP16> : bwd::fa_bwd_dq_kernel<D, FP16>;
  const unsigned bit = 1u << (4 + (D == 128 ? 4 : 0) + (FP16 ? 2 : 0) + (KV_SIDE ? 1 : 0));
  {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!(g_devices[dev].configured & bit)) {
      const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
      if (e != cudaSuccess) {
        set_error("cudaFuncSetAttribute(backward)", e);
        cudaGetLastError();
        return FA_ERR_CUDA;
      }
      g_devices[dev].configured |= bit;
    }
  }
  if (grid == 0) return FA_OK;
  kernel<<<static_cast<unsigned>(grid), bwd::kThreads, kSmem, stream>>>(x1, x2, y1, y2, prm);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_error(KV_SIDE ? "backward dK/dV launch" : "backward dQ launch", e);
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

// Backward shape: q, o, dout, dq [B, Nq, Hq, D]; k, v, dk, dv [B, Nk, Hkv, D]
// (dense: cu_q == nullptr), or packed sequences [total_q, Hq, D] and
// [total_k, Hkv, D] with device offsets cu_q, cu_k (Nq, Nk: upper bounds of
// the sequences' lengths).
struct BwdShape {
  const int* cu_q;
  const int* cu_k;
  int64_t B, Nq, Nk, Hq, Hkv, total_q, total_k;
};

BwdShape dense_bwd_shape(int64_t B, int64_t Nq, int64_t Nk, int64_t Hq, int64_t Hkv) {
  return BwdShape{nullptr, nullptr, B, Nq, Nk, Hq, Hkv, B * Nq, B * Nk};
}

template <int D, bool FP16>
fa_status bwd_run(int dev, const void* q, const void* k, const void* v, const void* o, const float* lse,
                  const void* dout, void* dq, void* dk, void* dv, const BwdShape& sh, float scale, int causal,
                  void* workspace, cudaStream_t stream) {
  const int64_t B = sh.B, Nq = sh.Nq, Nk = sh.Nk, Hq = sh.Hq, Hkv = sh.Hkv;
  const int64_t tq_rows = sh.total_q, tk_rows = sh.total_k;
  const int64_t n_qt = (Nq + kTile - 1) / kTile;
  const int64_t n_kt = (Nk + kTile - 1) / kTile;
  const int64_t npad = n_qt * kTile;
  const int64_t BHq = B * Hq;
  float* ws_d = static_cast<float*>(workspace);
  float* ws_l = reinterpret_cast<float*>(static_cast<char*>(workspace) + align256(static_cast<size_t>(BHq * npad) * 4));
  int* sched = reinterpret_cast<int*>(static_cast<char*>(workspace) + 2 * align256(static_cast<size_t>(BHq * npad) * 4));
  constexpr int64_t kPrepRows = 256 / (D / 8);  // rows per preprocess block
  const int64_t real_blocks = (tq_rows * Hq + kPrepRows - 1) / kPrepRows;
  const int64_t pad_blocks = sh.cu_q ? (BHq * npad + 255) / 256 : (BHq * (npad - Nq) + 255) / 256;
  if (real_blocks + pad_blocks > 0) {
    const unsigned grid = static_cast<unsigned>(real_blocks + pad_blocks);
    if (sh.cu_q) {
      bwd::fa_bwd_prep_varlen_kernel<D, FP16><<<grid, 256, 0, stream>>>(
          static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse, ws_d, ws_l, sh.cu_q,
          static_cast<int>(B), static_cast<int>(Hq), static_cast<int>(tq_rows), static_cast<int>(npad),
          static_cast<unsigned>(real_blocks), sched);
    } else {
      // a few blocks per SM striding over (b, h, rows) items
      const int64_t items = BHq * ((Nq + bwd::prep_rows_per_iter<D>() - 1) / bwd::prep_rows_per_iter<D>());
      const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(items, 8 * static_cast<int64_t>(device_sm_count(dev))));
      bwd::fa_bwd_prep_kernel<D, FP16><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
          static_cast<const uint16_t*>(o), static_cast<const uint16_t*>(dout), lse, ws_d, ws_l, static_cast<int>(B),
          static_cast<int>(Nq), static_cast<int>(Hq), static_cast<int>(npad), sched);
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
      set_error("backward preprocess launch", e);
      return FA_ERR_CUDA;
    }
  } else {
    const cudaError_t e = cudaMemsetAsync(sched, 0, 2 * sizeof(int), stream);  // no rows to preprocess
    if (e != cudaSuccess) {
      set_error("cudaMemsetAsync(backward work-item counters)", e);
      return FA_ERR_CUDA;
    }
  }
  const bool fp16 = FP16;
  // With no queries (or no keys) nothing is ever loaded from that side; its
  // maps only need a valid, aligned base.
  const void* qb = tq_rows > 0 ? q : k;
  const void* dob = tq_rows > 0 ? dout : k;
  const void* kb = tk_rows > 0 ? k : q;
  const void* vb = tk_rows > 0 ? v : q;
  CUtensorMap tq, tk, tv, tdo;
  if (make_tmap(&tq, qb, tq_rows > 0 ? tq_rows : 1, tq_rows > 0 ? Hq : 1, D, fp16) != FA_OK ||
      make_tmap(&tdo, dob, tq_rows > 0 ? tq_rows : 1, tq_rows > 0 ? Hq : 1, D, fp16) != FA_OK ||
      make_tmap(&tk, kb, tk_rows > 0 ? tk_rows : 1, tk_rows > 0 ? Hkv : 1, D, fp16) != FA_OK ||
      make_tmap(&tv, vb, tk_rows > 0 ? tk_rows : 1, tk_rows > 0 ? Hkv : 1, D, fp16) != FA_OK)
    return FA_ERR_CUDA;
  bwd::Params prm;
  prm.cu_q = sh.cu_q;
  prm.cu_k = sh.cu_k;
  prm.total_q = static_cast<int>(tq_rows);
  prm.total_k = static_cast<int>(tk_rows);
  prm.ws_d = ws_d;
  prm.ws_l = ws_l;
  prm.Nq = static_cast<int>(Nq);
  prm.Nk = static_cast<int>(Nk);
  prm.Hq = static_cast<int>(Hq);
  prm.Hkv = static_cast<int>(Hkv);
  prm.G = static_cast<int>(Hq / Hkv);
  prm.Npad = static_cast<int>(npad);
  // same base-2 factor as the forward (see launch)
  float c = scale * 1.44269504088896340736f;
  if (std::fabs(c) < FLT_MIN) c = std::signbit(c) ? -FLT_MIN : FLT_MIN;
  prm.scale_log2 = c;
  prm.scale = scale;
  prm.causal = causal ? 1 : 0;
  prm.wait_limit_ns = kDefaultWaitLimitNs;
  // rows are D * 2 bytes apart (a multiple of 128): 32-byte stores if the bases allow
  auto aligned32 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; };
  // persistent grids: one CTA per SM, at most one per work item
  const int64_t sms = device_sm_count(dev);
  // query side: work items (query tile, b, query head)
  prm.out0 = static_cast<uint16_t*>(dq);
  prm.out1 = nullptr;
  prm.BH = static_cast<int>(BHq);
  prm.n_tiles = static_cast<int>(n_qt);
  prm.n_items = static_cast<int>(n_qt * BHq);
  prm.sched = sched;
  prm.wide_stores = aligned32(dq) ? 1 : 0;
  fa_status st = bwd_launch<D, FP16, false>(dev, tq, tdo, tk, tv, prm, std::min<int64_t>(prm.n_items, sms), stream);
  if (st != FA_OK) return st;
  // key side: work items (key tile, b, K/V head)
  prm.out0 = static_cast<uint16_t*>(dk);
  prm.out1 = static_cast<uint16_t*>(dv);
  prm.BH = static_cast<int>(B * Hkv);
  prm.n_tiles = static_cast<int>(n_kt);
  prm.n_items = static_cast<int>(n_kt * B * Hkv);
  prm.sched = sched + 1;
  prm.wide_stores = aligned32(dk) && aligned32(dv) ? 1 : 0;
  st = bwd_launch<D, FP16, true>(dev, tk, tv, tq, tdo, prm, std::min<int64_t>(prm.n_items, sms), stream);
  if (st != FA_OK) return st;
  if (debug_enabled())
    std::fprintf(stderr, "[fa] bwd D=%d %s B=%lld Nq=%lld Nk=%lld Hq=%lld Hkv=%lld %s causal=%d items=%lld+%lld on %lld SMs\n",
                 D, FP16 ? "fp16" : "bf16", (long long)B, (long long)Nq, (long long)Nk, (long long)Hq, (long long)Hkv,
                 sh.cu_q ? "packed" : "dense", causal, (long long)(n_qt * BHq), (long long)(n_kt * B * Hkv),
                 (long long)sms);
  return FA_OK;
}

fa_status bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                   void* dq, void* dk, void* dv, const BwdShape& sh, int64_t D, float scale, int causal,
                   fa_dtype dtype, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  const int64_t B = sh.B, Nq = sh.Nq, Nk = sh.Nk, Hq = sh.Hq, Hkv = sh.Hkv;
  const int64_t tq_rows = sh.total_q, tk_rows = sh.total_k;
  if (B < 0 || Nq < 0 || Nk < 0 || Hq < 0 || Hkv < 0 || tq_rows < 0 || tk_rows < 0) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (Hq > 0 && (Hkv < 1 || Hq % Hkv != 0)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (B == 0 || Hq == 0 || (tq_rows == 0 && tk_rows == 0)) return FA_OK;
  if (tq_rows > 0 && (!q || !o || !lse || !dout || !dq)) return FA_ERR_INVALID_ARG;
  if (tk_rows > 0 && (!k || !v || !dk || !dv)) return FA_ERR_INVALID_ARG;
  if (sh.cu_q && !sh.cu_k) return FA_ERR_INVALID_ARG;
  const int64_t n_qt = (Nq + kTile - 1) / kTile, n_kt = (Nk + kTile - 1) / kTile;
  if (tq_rows > INT32_MAX - 2 * kTile || tk_rows > INT32_MAX - 2 * kTile || Nq > INT32_MAX - 2 * kTile ||
      Nk > INT32_MAX - 2 * kTile || Hq > INT32_MAX || B * Hq > INT32_MAX / (n_qt + 1) ||
      B * Hkv > INT32_MAX / (n_kt + 1))
    return FA_ERR_UNSUPPORTED;
  if (static_cast<double>(tq_rows) * Hq * D * 2 >= 1099511627776.0 ||
      static_cast<double>(tk_rows) * Hkv * D * 2 >= 1099511627776.0)
    return FA_ERR_UNSUPPORTED;
  // preprocess grid: total_q Hq / 16 row blocks plus at most B Hq Npad / 256 pad blocks stay below 2^31
  if ((tq_rows * Hq + B * Hq * (n_qt * kTile)) / 15 >= INT32_MAX) return FA_ERR_UNSUPPORTED;
  const size_t need = bwd_ws_bytes(B, Nq, Hq);
  if (workspace_bytes < need || (need > 0 && !workspace)) return FA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv), static_cast<const void*>(lse)})
    if (!aligned16(ptr)) return FA_ERR_MISALIGNED;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_MISALIGNED;
  int dev = 0;
  fa_status st = check_device(&dev);
  if (st != FA_OK) return st;
  st = load_encoder();
  if (st != FA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool fp16 = dtype == FA_FP16;
  if (D == 128)
    return fp16 ? bwd_run<128, true>(dev, q, k, v, o, lse, dout, dq, dk, dv, sh, scale, causal, workspace, s)
                : bwd_run<128, false>(dev, q, k, v, o, lse, dout, dq, dk, dv, sh, scale, causal, workspace, s);
  return fp16 ? bwd_run<64, true>(dev, q, k, v, o, lse, dout, dq, dk, dv, sh, scale, causal, workspace, s)
              : bwd_run<64, false>(dev, q, k, v, o, lse, dout, dq, dk, dv, sh, scale, causal, workspace, s);
}

}  // namespace

// ---------------------------------------------------------------- no-allocation scratch
// Scratch for fa_fwd_splitkv_noalloc: a fixed-size buffer compiled into the
// library, so that entry point needs no device allocation at all. Every GPU
// that loads the library holds it (kNoAllocScratchBytes) until the process
// exits. In host code `g_noalloc_scratch` only names the symbol; its device
// address is looked up per device below.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};
}  // namespace

// Device address of the scratch on the current device `dev`, looked up once per
// device (cudaGetSymbolAddress; no allocation) and cached.
fa_status noalloc_scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      set_error("cudaGetSymbolAddress(scratch)", e);
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return FA_OK;
}

// Synchronise `s`, then read and clear the status word (fa_status_sync).
fa_status sync_status(cudaStream_t s) {
  unsigned int word = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) {
    set_error("cudaStreamSynchronize", cudaGetLastError());
    return FA_ERR_CUDA;
  }
  if (cudaMemcpyFromSymbolAsync(&word, g_status_word, sizeof(word), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    set_error("reading the status word", cudaGetLastError());
    return FA_ERR_CUDA;
  }
  if (word == 0) return FA_OK;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbolAsync(g_status_word, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    set_error("clearing the status word", cudaGetLastError());
    return FA_ERR_CUDA;
  }
  if (word & 1u) return FA_ERR_TIMEOUT;
  if (word & 2u) return FA_ERR_INVALID_ARG;
  return FA_ERR_DEVICE_CHECK;
}

// Common exit of the entry points: with the debug switch on, a call that
// enqueued work waits for it and returns the device-side status itself.
fa_status finish(fa_status st, fa_stream_t stream, const char* what) {
  if (st != FA_OK || !debug_enabled()) return st;
  const fa_status dev = sync_status(reinterpret_cast<cudaStream_t>(stream));
  if (dev != FA_OK) std::fprintf(stderr, "[fa] %s: device status %d after the call\n", what, static_cast<int>(dev));
  return dev;
}

}  // namespace fa

extern "C" {

const char* fa_last_error(void) { return fa::g_last_error; }

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: null pointer, negative size, unknown dtype or non-finite scale";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: head dim not 64/128, size limit, or device is not sm_100";
    case FA_ERR_MISALIGNED: return "FA_ERR_MISALIGNED: a base pointer is not 16-byte aligned";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: a CUDA runtime call failed";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a device-side wait ran out; outputs are invalid";
    case FA_ERR_DEVICE_CHECK: return "FA_ERR_DEVICE_CHECK: a device-side index check failed; outputs are invalid";
  }
  return "FA_ERR_UNKNOWN";
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t N, int64_t H,
                 int64_t D, float scale, int causal, fa_dtype dtype, fa_stream_t stream) {
  try {
    return fa::finish(fa::fwd_impl(q, k, v, o, lse, fa::dense_shape(B, N, N, H, H, D), scale, causal, dtype, stream, 0, 0),
                      stream, "fa_fwd");
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

fa_status fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t Nq,
                     int64_t Nk, int64_t Hq, int64_t Hkv, int64_t D, float scale, int causal, fa_dtype dtype,
                     fa_stream_t stream) {
  try {
    return fa::finish(
        fa::fwd_impl(q, k, v, o, lse, fa::dense_shape(B, Nq, Nk, Hq, Hkv, D), scale, causal, dtype, stream, 0, 0), stream,
        "fa_fwd_gqa");
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* cu_seqlens_q,
                        const int32_t* cu_seqlens_k, int64_t B, int64_t max_seqlen_q, int64_t total_q, int64_t total_k,
                        int64_t Hq, int64_t Hkv, int64_t D, float scale, int causal, fa_dtype dtype,
                        fa_stream_t stream) {
  try {
    if (!cu_seqlens_q || !cu_seqlens_k) return FA_ERR_INVALID_ARG;
    fa::Shape sh{cu_seqlens_q, cu_seqlens_k, B, 0, 0, total_q, total_k, max_seqlen_q, Hq, Hkv, D};
    return fa::finish(fa::fwd_impl(q, k, v, o, lse, sh, scale, causal, dtype, stream, 0, 0), stream, "fa_fwd_varlen");
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

fa_status fa_fwd_splitkv_plan(int64_t B, int64_t Nq, int64_t Nk, int64_t Hq, int64_t Hkv, int64_t D, int num_splits,
                              int* splits_out, size_t* workspace_bytes) {
  try {
    if (!splits_out || !workspace_bytes || B < 0 || Nq < 0 || Nk < 0 || Hq < 0 || Hkv < 0 || num_splits < 0)
      return FA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
      cudaGetLastError();
      dev = -1;
    }
    const int sms = dev >= 0 ? fa::device_sm_count(dev) : 148;
    int tiles = 0;
    const int splits = fa::resolve_splits(num_splits, B, Nq, Nk, Hq, Hkv, sms, &tiles);
    *splits_out = splits;
    *workspace_bytes = splits > 1 ? fa::splitkv_bytes(splits, B * Hq, Nq, D) : 0;
    return FA_OK;
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

fa_status fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t Nq,
                         int64_t Nk, int64_t Hq, int64_t Hkv, int64_t D, float scale, int causal, fa_dtype dtype,
                         int num_splits, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  try {
    fa::Shape sh = fa::dense_shape(B, Nq, Nk, Hq, Hkv, D);
    if (num_splits < 0) return FA_ERR_INVALID_ARG;
    int splits = 1, tiles = 0;
    size_t need = 0;
    fa_status st = fa_fwd_splitkv_plan(B < 0 ? 0 : B, Nq < 0 ? 0 : Nq, Nk < 0 ? 0 : Nk, Hq < 0 ? 0 : Hq, Hkv < 0 ? 0 : Hkv,
                                       D, num_splits, &splits, &need);
    if (st != FA_OK) return st;
    if (splits > 1) {
      if (!workspace || workspace_bytes < need) return FA_ERR_INVALID_ARG;
      if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return FA_ERR_MISALIGNED;
      int dev = 0;
      cudaGetDevice(&dev);
      fa::resolve_splits(num_splits, B, Nq, Nk, Hq, Hkv, fa::device_sm_count(dev), &tiles);
      sh.n_splits = splits;
      sh.split_tiles = tiles;
      sh.part_o = static_cast<float*>(workspace);
      sh.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                             fa::align256(static_cast<size_t>(splits * B * Hq * Nq * D) * 4));
    }
    return fa::finish(fa::fwd_impl(q, k, v, o, lse, sh, scale, causal, dtype, stream, 0, 0), stream, "fa_fwd_splitkv");
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

fa_status fa_fwd_splitkv_noalloc(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B,
                                 int64_t Nq, int64_t Nk, int64_t Hq, int64_t Hkv, int64_t D, float scale, int causal,
                                 fa_dtype dtype, int num_splits, fa_stream_t stream) {
  try {
    if (num_splits < 0 || B < 0 || Nq < 0 || Nk < 0 || Hq < 0) return FA_ERR_INVALID_ARG;
    int splits = 1;
    size_t need = 0;
    fa_status st = fa_fwd_splitkv_plan(B, Nq, Nk, Hq, Hkv, D, num_splits, &splits, &need);
    if (st != FA_OK) return st;
    int requested = num_splits;
    // automatic count: fall back to the largest one whose partial results fit
    for (int r = splits - 1; num_splits == 0 && r >= 1 && need > fa::kNoAllocScratchBytes; --r) {
      st = fa_fwd_splitkv_plan(B, Nq, Nk, Hq, Hkv, D, r, &splits, &need);
      if (st != FA_OK) return st;
      requested = r;
    }
    if (need > fa::kNoAllocScratchBytes) {
      std::snprintf(fa::g_last_error, sizeof(fa::g_last_error),
                    "split-KV scratch of %zu bytes needed, the built-in scratch holds %zu bytes", need,
                    fa::kNoAllocScratchBytes);
      return FA_ERR_UNSUPPORTED;
    }
    fa::Shape sh = fa::dense_shape(B, Nq, Nk, Hq, Hkv, D);
    if (splits > 1) {
      int dev = 0;
      const cudaError_t e = cudaGetDevice(&dev);
      if (e != cudaSuccess) {
        fa::set_error("cudaGetDevice", e);
        cudaGetLastError();
        return FA_ERR_CUDA;
      }
      if (dev < 0 || dev >= fa::kMaxDevices) return FA_ERR_UNSUPPORTED;
      void* scratch = nullptr;
      st = fa::noalloc_scratch_address(dev, &scratch);
      if (st != FA_OK) return st;
      int tiles = 0;
      fa::resolve_splits(requested, B, Nq, Nk, Hq, Hkv, fa::device_sm_count(dev), &tiles);
      sh.n_splits = splits;
      sh.split_tiles = tiles;
      sh.part_o = static_cast<float*>(scratch);
      sh.part_lse = reinterpret_cast<float*>(static_cast<char*>(scratch) +
                                             fa::align256(static_cast<size_t>(splits * B * Hq * Nq * D) * 4));
    }
    return fa::finish(fa::fwd_impl(q, k, v, o, lse, sh, scale, causal, dtype, stream, 0, 0), stream,
                      "fa_fwd_splitkv_noalloc");
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

fa_status fa_fwd_debug(const void* q, const void* k, const void* v, void* o, float* lse, int64_t B, int64_t N,
                       int64_t H, int64_t D, float scale, int causal, fa_dtype dtype, fa_stream_t stream,
                       uint64_t wait_limit_ns, int withhold_v_load) {
  try {
    return fa::finish(fa::fwd_impl(q, k, v, o, lse, fa::dense_shape(B, N, N, H, H, D), scale, causal, dtype, stream,
                                    wait_limit_ns, withhold_v_load ? 1 : 0),
                      stream, "fa_fwd_debug");
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

fa_status fa_bwd_workspace_size(int64_t B, int64_t N, int64_t H, size_t* workspace_bytes) {
  if (!workspace_bytes || B < 0 || N < 0 || H < 0) return FA_ERR_INVALID_ARG;
  *workspace_bytes = fa::bwd_ws_bytes(B, N, H);
  return FA_OK;
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                 void* dq, void* dk, void* dv, int64_t B, int64_t N, int64_t H, int64_t D, float scale, int causal,
                 fa_dtype dtype, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  try {
    if (B < 0 || N < 0) return FA_ERR_INVALID_ARG;
    return fa::finish(fa::bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, fa::dense_bwd_shape(B, N, N, H, H), D, scale,
                                    causal, dtype, workspace, workspace_bytes, stream),
                      stream, "fa_bwd");
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

fa_status fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                     void* dq, void* dk, void* dv, int64_t B, int64_t Nq, int64_t Nk, int64_t Hq, int64_t Hkv,
                     int64_t D, float scale, int causal, fa_dtype dtype, void* workspace, size_t workspace_bytes,
                     fa_stream_t stream) {
  try {
    if (B < 0 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
    return fa::finish(fa::bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, fa::dense_bwd_shape(B, Nq, Nk, Hq, Hkv), D,
                                    scale, causal, dtype, workspace, workspace_bytes, stream),
                      stream, "fa_bwd_gqa");
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, const int32_t* cu_seqlens_q,
                        const int32_t* cu_seqlens_k, int64_t B, int64_t max_seqlen_q, int64_t max_seqlen_k,
                        int64_t total_q, int64_t total_k, int64_t Hq, int64_t Hkv, int64_t D, float scale, int causal,
                        fa_dtype dtype, void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  try {
    if (!cu_seqlens_q || !cu_seqlens_k) return FA_ERR_INVALID_ARG;
    const fa::BwdShape sh{cu_seqlens_q, cu_seqlens_k, B, max_seqlen_q, max_seqlen_k, Hq, Hkv, total_q, total_k};
    return fa::finish(fa::bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, sh, D, scale, causal, dtype, workspace,
                                    workspace_bytes, stream),
                      stream, "fa_bwd_varlen");
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

fa_status fa_status_sync(fa_stream_t stream) {
  try {
    return fa::sync_status(reinterpret_cast<cudaStream_t>(stream));
  } catch (...) {
    return FA_ERR_CUDA;
  }
}

}  // extern "C"
