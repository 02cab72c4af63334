// Host side of the C ABI (include/qlora.h): argument checks, the NF4 table,
// workspace planning, TMA descriptors and kernel launches. No allocation,
// no synchronisation (except qlora_device_status), no exceptions across the
// ABI.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>
#include <utility>

#include <cudaTypedefs.h>

#include "../../include/qlora.h"
#include "kernels.h"
#include "nf4_dev.cuh"
#include "ptx.cuh"

namespace qlora {
namespace {

constexpr int kBlock = 64;
constexpr int kGroup = 256;
constexpr int kMaxRank = 256;
constexpr int kGemvMaxM = 16;

// ------------------------------------------------------------------ NF4 table
double normal_cdf(double z) { return 0.5 * std::erfc(-z / std::sqrt(2.0)); }

// Phi^-1(p) for p in [1/2, 1) by Newton's method from z = 0. Phi is concave
// on z >= 0, so the iterates increase monotonically to the root.
double normal_quantile_upper(double p) {
  const double inv_sqrt_2pi = 0.39894228040143267794;
  double z = 0.0;
  for (int it = 0; it < 200; ++it) {
    const double f = normal_cdf(z) - p;
    const double d = inv_sqrt_2pi * std::exp(-0.5 * z * z);
    const double step = f / d;
    z -= step;
    if (std::fabs(step) <= 1e-17 * std::fmax(1.0, std::fabs(z))) break;
  }
  return z;
}

struct Tables {
  float cb[16];
  float mid[16];
  double cut[16];
  float cell_m[33];
  float cell_below[33];
};

const Tables& tables() {
  static Tables t = [] {
    Tables r{};
    const double delta = 0.5 * ((1.0 - 1.0 / 30.0) + (1.0 - 1.0 / 32.0));
    double lv[16];
    int n = 0;
    for (int j = 0; j < 7; ++j) lv[n++] = -normal_quantile_upper(delta + j * (0.5 - delta) / 7.0);
    lv[n++] = 0.0;
    for (int j = 0; j < 8; ++j) lv[n++] = normal_quantile_upper(delta + j * (0.5 - delta) / 8.0);
    // ascending order: the negatives grow toward 0 as j grows, the positives shrink
    double sorted[16];
    for (int i = 0; i < 7; ++i) sorted[i] = lv[i];          // j = 0..6: -1.x ... -0.1
    sorted[7] = 0.0;
    for (int i = 0; i < 8; ++i) sorted[8 + i] = lv[15 - i];  // j = 7..0
    const double top = normal_quantile_upper(delta);
    for (int i = 0; i < 16; ++i) r.cb[i] = static_cast<float>(sorted[i] / top);
    for (int i = 0; i < 15; ++i)
      r.mid[i] = static_cast<float>((static_cast<double>(r.cb[i]) + static_cast<double>(r.cb[i + 1])) / 2.0);
    r.mid[15] = 2.0f;
    for (int i = 0; i < 15; ++i)
      r.cut[i] = (static_cast<double>(r.mid[i]) + static_cast<double>(std::nextafter(r.mid[i], 2.0f))) / 2.0;
    r.cut[15] = 2.0;
    // encoder cells: cell c covers x in [(c - 16.5) / 16, (c - 15.5) / 16],
    // widened by twice the guard; at most one midpoint falls in a widened cell
    // (the midpoints are more than 0.08 apart, a cell is 0.0625 wide)
    const double g2 = 2.0 * static_cast<double>(kEncodeGuard);
    for (int c = 0; c <= 32; ++c) {
      const double lo = (c - 16.5) / 16.0 - g2, hi = (c - 15.5) / 16.0 + g2;
      int below = 0, cand = -1;
      for (int j = 0; j < 15; ++j) {
        if (r.mid[j] < lo) ++below;
        else if (r.mid[j] <= hi) cand = j;
      }
      r.cell_m[c] = cand >= 0 ? r.mid[cand] : 4.0f;
      r.cell_below[c] = static_cast<float>(below);
    }
    return r;
  }();
  return t;
}

// ------------------------------------------------------------------ device state
struct DevState {
  bool checked = false;
  bool ok = false;
  int sms = 148;
  bool attrs = false;      // kernel attributes set in context `ctx`
  CUcontext ctx = nullptr;
  int pair_clusters = 0;   // CTA pairs of k_tc_pair that can be resident at once
};
std::mutex g_mu;
DevState g_dev[64];

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

template <int BN, int AS, int BS>
cudaError_t set_small_attr() {
  return cudaFuncSetAttribute(k_tc_small<BN, AS, BS, small_stages(BN)>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              tc_small_smem_bytes<BN>());
}

template <int BN>
cudaError_t set_small_attrs() {
  cudaError_t e;
  if ((e = set_small_attr<BN, A_TMA_K, B_TMA_K>()) != cudaSuccess) return e;
  if ((e = set_small_attr<BN, A_TMA_K, B_TMA_MN>()) != cudaSuccess) return e;
  return set_small_attr<BN, A_TMA_MN, B_TMA_MN>();
}

template <int AS, int NH>
cudaError_t pair_clusters_of(int* out) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(448, 1, 1);
  cfg.dynamicSmemBytes = tc_pair_smem_bytes(NH);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaFuncSetAttribute(k_tc_pair<AS, NH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       tc_pair_smem_bytes(NH));
  if (e != cudaSuccess) return e;
  return cudaOccupancyMaxActiveClusters(out, k_tc_pair<AS, NH>, &cfg);
}

// How many 2-CTA clusters of the pair kernels fit on the device at once (one
// CTA per SM, clusters confined to a GPC); also sets their shared-memory limit.
cudaError_t pair_clusters(int* out) {
  int n[4] = {0, 0, 0, 0};
  cudaError_t e;
  if ((e = pair_clusters_of<A_DQ_K, 1>(&n[0])) != cudaSuccess) return e;
  if ((e = pair_clusters_of<A_DQ_K, 2>(&n[1])) != cudaSuccess) return e;
  if ((e = pair_clusters_of<A_DQ_MN, 1>(&n[2])) != cudaSuccess) return e;
  if ((e = pair_clusters_of<A_DQ_MN, 2>(&n[3])) != cudaSuccess) return e;
  *out = std::min(std::min(n[0], n[1]), std::min(n[2], n[3]));
  return (*out > 0) ? cudaSuccess : cudaErrorInvalidConfiguration;
}

}  // namespace

// The calling thread's current CUDA context, made current by the runtime if
// needed (cuCtxGetCurrent through the runtime's driver entry point, so the
// library needs no link-time dependency on the driver library).
CUcontext current_context() {
  using Fn = CUresult (*)(CUcontext*);
  static Fn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return static_cast<Fn>(nullptr);
    }
    return reinterpret_cast<Fn>(p);
  }();
  if (fn == nullptr) return nullptr;
  CUcontext c = nullptr;
  if (fn(&c) != CUDA_SUCCESS) return nullptr;
  if (c == nullptr) {
    // nothing has used the runtime on this thread yet: cudaSetDevice
    // initialises the device's primary context and makes it current
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    if (fn(&c) != CUDA_SUCCESS) return nullptr;
  }
  return c;
}

namespace {

qlora_status_t device_ready(int* sms_out, int* pairs_out = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QLORA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DevState& st = g_dev[dev];
  if (!st.checked) {
    st.checked = true;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return QLORA_ERR_CUDA;
    st.ok = (prop.major == 10 && prop.minor == 0);
    st.sms = prop.multiProcessorCount;
  }
  if (!st.ok) return QLORA_ERR_UNSUPPORTED_DEVICE;
  // kernel attributes belong to the context: set them again in a new one
  // (after cudaDeviceReset the runtime creates a new primary context)
  CUcontext ctx = current_context();
  if (ctx == nullptr) return QLORA_ERR_CUDA;
  if (st.attrs && st.ctx != ctx) st.attrs = false;
  if (!st.attrs) {
    cudaError_t e = pair_clusters(&st.pair_clusters);
    if (e == cudaSuccess) e = set_small_attrs<64>();
    if (e == cudaSuccess) e = set_small_attrs<128>();
    if (e == cudaSuccess) e = set_small_attrs<192>();
    if (e == cudaSuccess) e = set_small_attrs<256>();
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_merge_lora, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(merge_smem_bytes(kMaxRank)));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(k_merge_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(merge_tc_smem_bytes()));
    if (e != cudaSuccess) return QLORA_ERR_CUDA;
    st.attrs = true;
    st.ctx = ctx;
  }
  if (sms_out) *sms_out = st.sms;
  if (pairs_out) *pairs_out = st.pair_clusters;
  return QLORA_OK;
}

}  // namespace

// The same device check every entry point runs first (see device_ready), for
// the entry points defined in other files.
int check_current_device_status() { return static_cast<int>(device_ready(nullptr)); }

namespace {

// ------------------------------------------------------------------ helpers
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t rup(int64_t a, int64_t b) { return cdiv(a, b) * b; }
inline int32_t r64_of(int32_t r) { return static_cast<int32_t>(rup(r, 64)); }
inline size_t al256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

bool map2d(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t inner, uint64_t outer,
           uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// bf16 [outer x inner] row-major, 128-byte swizzled boxes of {64, box_outer}
bool map_bf16(CUtensorMap* m, const void* ptr, int64_t outer, int64_t inner, int64_t ld, uint32_t box_outer) {
  return map2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, inner, outer, ld * 2, 64, box_outer,
               CU_TENSOR_MAP_SWIZZLE_128B);
}

// Split count for a reduction of `ktiles` 64-wide k-tiles over `tiles`
// output tiles of 128 x r64 on `sms` persistent CTAs. The estimate is the
// bytes the busiest CTA moves: its tiles times (their k-tiles of operand
// loads + one fp32 partial tile written), plus its share of the reduction's
// re-read of all partial slabs.
int pick_splits(int64_t tiles, int64_t ktiles, int32_t r64, int sms) {
  tiles = std::max<int64_t>(1, tiles);
  const double load = 16384.0 + 128.0 * r64;  // bytes per k-tile
  const double tile_out = 512.0 * r64;        // fp32 partial tile
  int best = 1;
  double best_cost = 1e300;
  for (int s = 1; s <= 16 && s <= ktiles; ++s) {
    const double per_cta = static_cast<double>(cdiv(tiles * s, sms));
    const double cost = per_cta * (static_cast<double>(cdiv(ktiles, s)) * load + tile_out) +
                        static_cast<double>(s * tiles) * tile_out / sms;
    if (cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  const int64_t per = cdiv(ktiles, best);
  return static_cast<int>(cdiv(ktiles, per));
}

struct SmallPlan {
  int splits, kt_split;
  int64_t rows_pad;
  size_t part_bytes;
};

SmallPlan plan_small(int64_t rows, int64_t ktiles, int32_t r64, int sms) {
  SmallPlan p;
  const int64_t tiles = cdiv(rows, 128);
  p.splits = pick_splits(tiles, ktiles, r64, sms);
  p.kt_split = static_cast<int>(cdiv(ktiles, p.splits));
  p.rows_pad = tiles * 128;
  p.part_bytes = static_cast<size_t>(p.splits) * p.rows_pad * r64 * sizeof(float);
  return p;
}

// Token groups of 256 per restored weight tile: two once there are more than
// 256 tokens (each restored tile then feeds 512 tokens), else one.
inline int pair_nh(int64_t m) { return m > 256 ? 2 : 1; }

// Stream-K slots of the pair kernels: one fp32 [128 x 256 NH] partial per CTA
// (at most one CTA per SM) and four flags per CTA.
inline size_t sk_part_bytes(int64_t m, int sms) {
  return static_cast<size_t>(sms) * 128 * 256 * pair_nh(m) * sizeof(float);
}
inline size_t sk_flag_bytes(int sms) { return static_cast<size_t>(sms) * 4 * sizeof(uint32_t); }

// Pair tiles of the forward (features = d_out) or dX (features = d_in).
inline int64_t pair_tiles(int64_t m, int64_t features) {
  return cdiv(features, 256) * cdiv(m, 256 * pair_nh(m));
}

// GEMM schedule setting (qlora_sched_t) and the automatic rule: stream-K for
// reductions of at least kSkMinKtiles k-tiles.
std::atomic<int> g_sched{QLORA_SCHED_AUTO};
constexpr int64_t kSkMinKtiles = 128;
inline bool sk_wanted(int64_t kt_main, int mode) {
  return mode == QLORA_SCHED_STREAM_K || (mode == QLORA_SCHED_AUTO && kt_main >= kSkMinKtiles);
}

struct WsPlan {
  size_t u_pad, v_pad, b_pad, dy_pad, part, total;
  bool sk_ok;        // a pair GEMM of the call may use the stream-K schedule
  size_t sk_total;   // total with room for the stream-K slots and flags (>= total)
  size_t flags_off;  // stream-K flags (sk_total plan), from the 256-aligned workspace start
};

// Workspace layout: [u_pad][v_pad][b_pad][dy_pad][split partials][flags],
// each 256-aligned. The forward needs no v_pad, no dy_pad and only the x A^T
// partials. dy_pad holds dY with its rows padded to a multiple of 8 elements
// when N % 8 != 0 (the TMA loads of dY need 16-byte row strides). The pair kernels'
// stream-K slots reuse the partials region (it is free while they run), which
// grows to hold them in the sk_total plan; their flags get a region of their
// own, zeroed at the start of the call, before any kernel of the call runs:
// `total` is what a call needs, `sk_total` what lets it use the stream-K
// schedule when that pays.
WsPlan plan_ws(int64_t m, int64_t n, int64_t k, int32_t r, int sms, bool fwd_only, int mode) {
  const int32_t r64 = r64_of(r);
  WsPlan w{};
  w.u_pad = al256(static_cast<size_t>(m) * r64 * 2);
  w.v_pad = fwd_only ? 0 : al256(static_cast<size_t>(m) * r64 * 2);
  w.b_pad = (r % 8 != 0) ? al256(static_cast<size_t>(n) * r64 * 2) : 0;
  w.dy_pad = (!fwd_only && n % 8 != 0) ? al256(static_cast<size_t>(m) * rup(n, 8) * 2) : 0;
  size_t part = plan_small(m, cdiv(k, 64), r64, sms).part_bytes;  // x A^T
  if (!fwd_only) {
    part = std::max(part, plan_small(m, cdiv(n, 64), r64, sms).part_bytes);  // dY B
    part = std::max(part, plan_small(k, cdiv(m, 64), r64, sms).part_bytes);  // dA
    part = std::max(part, plan_small(n, cdiv(m, 64), r64, sms).part_bytes);  // dB
  }
  w.part = al256(part);
  w.total = w.u_pad + w.v_pad + w.b_pad + w.dy_pad + w.part + 256;
  // the forward reduces over K, dX over N; slots only where stream-K may run
  const int64_t tiles = std::max(sk_wanted(cdiv(k, 64), mode) ? pair_tiles(m, n) : int64_t(0),
                                 fwd_only || !sk_wanted(cdiv(n, 64), mode) ? int64_t(0) : pair_tiles(m, k));
  w.sk_ok = m > kGemvMaxM && tiles > sms / 4;
  w.flags_off = w.u_pad + w.v_pad + w.b_pad + w.dy_pad + std::max(w.part, al256(sk_part_bytes(m, sms)));
  w.sk_total = w.sk_ok ? w.flags_off + al256(sk_flag_bytes(sms)) + 256 : w.total;
  return w;
}

qlora_status_t check_nf4(const qlora_nf4_t* q) {
  if (q == nullptr || q->codes == nullptr || q->absmax == nullptr) return QLORA_ERR_INVALID_ARG;
  if (q->block != kBlock || (q->dq_group != kGroup && q->dq_group != 0)) return QLORA_ERR_INVALID_ARG;
  if (q->dq_group == kGroup && q->scale_codes == nullptr) return QLORA_ERR_INVALID_ARG;
  if (q->dq_group == kGroup && (q->dq_code < QLORA_DQ_U8_256 || q->dq_code > QLORA_DQ_S8_MID))
    return QLORA_ERR_INVALID_ARG;
  if (q->reserved != 0) return QLORA_ERR_INVALID_ARG;
  if (q->n_out <= 0 || q->k_in <= 0 || q->k_in % kBlock != 0) return QLORA_ERR_SHAPE;
  if (q->n_out > (int64_t(1) << 31) - 1 || q->k_in > (int64_t(1) << 31) - 1) return QLORA_ERR_SHAPE;
  if (!aligned16(q->codes)) return QLORA_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(q->absmax) & 3u) != 0) return QLORA_ERR_ALIGNMENT;
  return QLORA_OK;
}

std::atomic<uint64_t> g_launches{0};

// Every kernel launch is followed by this check; it also counts the launch.
inline qlora_status_t launch_status() {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cudaGetLastError() == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

CUtensorMap zero_map() {
  CUtensorMap m;
  std::memset(&m, 0, sizeof(m));
  return m;
}

// Launch as a programmatic dependent of the kernel in front on the stream:
// the kernel itself waits for that grid before touching global memory (every
// kernel launched this way calls grid_dependency_wait first), so stream order
// holds while the launch and the kernel's set-up overlap the one in front.
template <typename... KArgs, typename... Args>
qlora_status_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return launch_status();
}

// Zero-padded copy of a [rows x r] bf16 matrix into [rows x r64].
qlora_status_t pad_cols(const __nv_bfloat16* src, __nv_bfloat16* dst, int64_t rows, int32_t r, int32_t r64, int sms,
                        cudaStream_t st) {
  const unsigned blocks = static_cast<unsigned>(std::min<int64_t>(cdiv(rows * r64, 256), int64_t(sms) * 8));
  return launch_pdl(k_pad_cols, dim3(std::max(blocks, 1u)), dim3(256), 0, st, src, dst, rows, r, r64);
}

// Persistent launch: one CTA per SM at most, each walking the tile list.
template <int BN, int AS, int BS>
qlora_status_t launch_small_bn(int sms, cudaStream_t st, const CUtensorMap& a, const CUtensorMap& b,
                               const SmallParams& p) {
  const int64_t tiles = static_cast<int64_t>(p.tiles) * p.splits;
  if (tiles <= 0) return QLORA_ERR_SHAPE;
  const unsigned grid = static_cast<unsigned>(std::min<int64_t>(tiles, sms));
  return launch_pdl(k_tc_small<BN, AS, BS, small_stages(BN)>, dim3(grid), dim3(192), tc_small_smem_bytes<BN>(), st,
                    a, b, p);
}

// Persistent CTA-pair launch: at most `pairs` clusters of two CTAs.
template <int AS, int NH>
qlora_status_t launch_pair_nh(int pairs, cudaStream_t st, const CUtensorMap& b, const CUtensorMap& bl,
                              const CUtensorMap& c, const CUtensorMap& o, const TcParams& p) {
  const int64_t tiles = static_cast<int64_t>(p.tiles_rows) * p.tiles_cols;
  if (tiles <= 0 || pairs <= 0) return QLORA_ERR_SHAPE;
  const unsigned nclusters = static_cast<unsigned>(std::min<int64_t>(tiles, pairs));
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // a programmatic dependent of the kernel in front (the pair kernel waits
  // for it before touching global memory)
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(2 * nclusters, 1, 1);
  cfg.blockDim = dim3(448, 1, 1);
  cfg.dynamicSmemBytes = tc_pair_smem_bytes(NH);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k_tc_pair<AS, NH>, b, bl, c, o, p);
  if (e != cudaSuccess) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return launch_status();
}

// Features per tile of a data-parallel forward: of the widths 256, 240, ...,
// 128 (multiples of 16: each CTA of a pair restores half, in 8-row swizzle
// atoms) the one that needs the fewest features per pair over all waves,
// ceil(tiles / pairs) * width, i.e. the one whose last wave is fullest; ties
// go to the wider tile.
int32_t pick_feat_n(int64_t features, int64_t tiles_cols, int pairs) {
  int32_t best = 256;
  int64_t best_cost = cdiv(cdiv(features, 256) * tiles_cols, pairs) * 256;
  for (int32_t fn = 240; fn >= 128; fn -= 16) {
    const int64_t cost = cdiv(cdiv(features, fn) * tiles_cols, pairs) * fn;
    if (cost < best_cost) {
      best = fn;
      best_cost = cost;
    }
  }
  return best;
}

// The output [m x features] bf16 (row stride p.ldo) is written through TMA
// stores when its row stride is a multiple of 16 bytes.
//
// Stream-K: with `sk_region` (the workspace's partials region, holding at
// least the slots of sk_part_bytes) and `sk_flags` (sk_flag_bytes, zeroed by
// the caller before the call's first kernel), and a tile count above the
// pair count that leaves the last wave partly idle, the pairs split the work
// evenly (see k_tc_pair).
template <int AS>
qlora_status_t launch_pair(int pairs, int64_t m, cudaStream_t st, const CUtensorMap& b, const CUtensorMap& bl,
                           const CUtensorMap& c, TcParams p, uint8_t* sk_region, uint32_t* sk_flags, int sms,
                           int mode) {
  CUtensorMap o = zero_map();
  p.tma_out = 0;
  if (p.ldo % 8 == 0 && (reinterpret_cast<uintptr_t>(p.out) & 15u) == 0) {
    if (!map2d(&o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, p.out, static_cast<uint64_t>(p.rows), static_cast<uint64_t>(m),
               static_cast<uint64_t>(p.ldo) * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
      return QLORA_ERR_CUDA;
    p.tma_out = 1;
  }
  // the signed scale code's two group constants need the NH = 1 restore slots
  const int nh = (p.dq && p.dqc == QLORA_DQ_S8_MID) ? 1 : pair_nh(m);
  p.tiles_cols = static_cast<int32_t>(cdiv(m, 256 * nh));
  p.feat_n = 256;
  p.tiles_rows = static_cast<int32_t>(cdiv(p.rows, 256));
  const int64_t tiles = static_cast<int64_t>(p.tiles_rows) * p.tiles_cols;
  p.sk = 0;
  p.sk_part = nullptr;
  p.sk_flags = nullptr;
  if (sk_region != nullptr && sk_flags != nullptr && sk_wanted(p.kt_main, mode) && p.tma_out && pairs > 1 &&
      2 * pairs <= sms && tiles > pairs && tiles % pairs != 0) {
    p.sk = 1;
    p.sk_part = reinterpret_cast<float*>(sk_region);
    p.sk_flags = sk_flags;
  }
  if (AS == A_DQ_K && !p.sk && pairs > 0) {
    p.feat_n = pick_feat_n(p.rows, p.tiles_cols, pairs);
    p.tiles_rows = static_cast<int32_t>(cdiv(p.rows, p.feat_n));
  }
  if (nh == 2) return launch_pair_nh<AS, 2>(pairs, st, b, bl, c, o, p);
  return launch_pair_nh<AS, 1>(pairs, st, b, bl, c, o, p);
}

template <int AS, int BS>
qlora_status_t launch_small(int32_t r64, int sms, cudaStream_t st, const CUtensorMap& a, const CUtensorMap& b,
                            const SmallParams& p) {
  switch (r64) {
    case 64: return launch_small_bn<64, AS, BS>(sms, st, a, b, p);
    case 128: return launch_small_bn<128, AS, BS>(sms, st, a, b, p);
    case 192: return launch_small_bn<192, AS, BS>(sms, st, a, b, p);
    case 256: return launch_small_bn<256, AS, BS>(sms, st, a, b, p);
    default: return QLORA_ERR_SHAPE;
  }
}

// A TMA-fed LoRA product over a reduction of length `kdim`: split-K partial
// slabs in `part`, then the fixed-order reduction writes mode 0 bf16(scale *
// .) to out_pad [rows x r64] (and out_c [rows x r] when set), mode 1 fp32
// out_f [rows x r], mode 2 fp32 out_f [r x rows] (transposed). With one
// split the GEMM's drain writes the result and no reduction is launched.
template <int AS, int BS>
qlora_status_t lora_product(const CUtensorMap& ma, const CUtensorMap& mb, int64_t rows, int64_t kdim,
                            int32_t r, float scale, int mode, __nv_bfloat16* out_pad, __nv_bfloat16* out_c,
                            float* out_f, float* part, int sms, cudaStream_t st) {
  const int32_t r64 = r64_of(r);
  const SmallPlan sp = plan_small(rows, cdiv(kdim, 64), r64, sms);
  SmallParams p{};
  p.rows = static_cast<int32_t>(rows);
  p.rows_pad = static_cast<int32_t>(sp.rows_pad);
  p.ld = r64;
  p.cols = r;
  p.tiles = static_cast<int32_t>(cdiv(rows, 128));
  p.kt_main = static_cast<int32_t>(cdiv(kdim, 64));
  p.kt_split = sp.kt_split;
  p.splits = sp.splits;
  p.part = part;
  p.scale = scale;
  p.mode = mode;
  p.out_pad = out_pad;
  p.out_c = out_c;
  p.out_f = out_f;
  qlora_status_t s = launch_small<AS, BS>(r64, sms, st, ma, mb, p);
  if (s != QLORA_OK || p.splits == 1) return s;   // one split: the GEMM wrote the result itself
  const int total = p.rows * (r64 / 4);
  const int blocks = static_cast<int>(std::min<int64_t>(cdiv(total, 256), int64_t(sms) * 8));
  return launch_pdl(k_reduce_splits, dim3(std::max(blocks, 1)), dim3(256), 0, st, p);
}

struct LinearArgs {
  const qlora_nf4_t* q;
  int64_t m;
  int32_t r;
  float alpha;
  void* ws;
  size_t ws_bytes;
};

qlora_status_t check_linear(const LinearArgs& a, int sms, bool fwd_only) {
  qlora_status_t s = check_nf4(a.q);
  if (s != QLORA_OK) return s;
  if (a.m < 0 || a.m > (int64_t(1) << 31) - 1) return QLORA_ERR_SHAPE;
  if (a.r < 1 || a.r > kMaxRank) return QLORA_ERR_SHAPE;
  if (!std::isfinite(a.alpha)) return QLORA_ERR_INVALID_ARG;
  if (a.m == 0) return QLORA_OK;
  if (a.ws == nullptr || !aligned16(a.ws)) return a.ws == nullptr ? QLORA_ERR_WORKSPACE : QLORA_ERR_ALIGNMENT;
  if (a.ws_bytes < plan_ws(a.m, a.q->n_out, a.q->k_in, a.r, sms, fwd_only, QLORA_SCHED_DATA_PARALLEL).total)
    return QLORA_ERR_WORKSPACE;
  return QLORA_OK;
}

}  // namespace
}  // namespace qlora

using namespace qlora;

extern "C" {

int32_t qlora_version(void) { return 10200; }

uint64_t qlora_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

qlora_status_t qlora_set_gemm_schedule(int32_t mode) {
  if (mode != QLORA_SCHED_AUTO && mode != QLORA_SCHED_DATA_PARALLEL && mode != QLORA_SCHED_STREAM_K)
    return QLORA_ERR_INVALID_ARG;
  g_sched.store(mode);
  return QLORA_OK;
}

int32_t qlora_get_gemm_schedule(void) { return g_sched.load(); }

const char* qlora_status_string(qlora_status_t s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_SHAPE: return "unsupported shape";
    case QLORA_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100 (B200)";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_TIMEOUT: return "kernel gave up on a bounded wait";
  }
  return "unknown status";
}

qlora_status_t qlora_nf4_codebook(float out[16]) {
  if (out == nullptr) return QLORA_ERR_INVALID_ARG;
  std::memcpy(out, tables().cb, sizeof(float) * 16);
  return QLORA_OK;
}

size_t qlora_nf4_bytes_ex(int64_t n_out, int64_t k_in, int32_t dq_group, int32_t dq_code, size_t out[3]) {
  if (n_out <= 0 || k_in <= 0 || k_in % kBlock != 0 || (dq_group != kGroup && dq_group != 0)) return 0;
  if (dq_group == kGroup && (dq_code < QLORA_DQ_U8_256 || dq_code > QLORA_DQ_S8_MID)) return 0;
  const int64_t nb = n_out * k_in / kBlock;
  const bool dq = dq_group == kGroup;
  const size_t b0 = static_cast<size_t>(n_out * k_in / 2);
  const size_t b1 = dq ? static_cast<size_t>(nb) : 0;
  const int64_t per_group = (dq && dq_code == QLORA_DQ_S8_MID) ? 2 : 1;   // group constants
  const size_t b2 = static_cast<size_t>(dq ? per_group * cdiv(nb, kGroup) : nb) * sizeof(float);
  if (out) {
    out[0] = b0;
    out[1] = b1;
    out[2] = b2;
  }
  return b0 + b1 + b2;
}

size_t qlora_nf4_bytes(int64_t n_out, int64_t k_in, int32_t dq_group, size_t out[3]) {
  return qlora_nf4_bytes_ex(n_out, k_in, dq_group, QLORA_DQ_U8_256, out);
}

namespace {
int current_sms() {
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) sms = v;
  }
  cudaGetLastError();
  return sms;
}
}  // namespace

size_t qlora_workspace_bytes(int64_t m, int64_t n_out, int64_t k_in, int32_t r) {
  if (m < 0 || n_out <= 0 || k_in <= 0 || r < 1 || r > kMaxRank) return 0;
  // sized for the stream-K slots wherever any schedule setting could use
  // them, so the answer does not depend on the process-wide setting
  return plan_ws(std::max<int64_t>(m, 1), n_out, k_in, r, current_sms(), false, QLORA_SCHED_STREAM_K).sk_total;
}

size_t qlora_fwd_workspace_bytes(int64_t m, int64_t n_out, int64_t k_in, int32_t r) {
  if (m < 0 || n_out <= 0 || k_in <= 0 || r < 1 || r > kMaxRank) return 0;
  return plan_ws(std::max<int64_t>(m, 1), n_out, k_in, r, current_sms(), true, QLORA_SCHED_DATA_PARALLEL).total;
}

qlora_status_t qlora_quantize_nf4(const void* w_bf16, const qlora_nf4_t* q, void* stream) {
  qlora_status_t s = check_nf4(q);
  if (s != QLORA_OK) return s;
  if (w_bf16 == nullptr) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(w_bf16)) return QLORA_ERR_ALIGNMENT;
  if ((s = device_ready(nullptr)) != QLORA_OK) return s;
  const int64_t nb = q->n_out * q->k_in / kBlock;
  QuantParams qp{};
  std::memcpy(qp.cut, tables().cut, sizeof(qp.cut));
  std::memcpy(qp.cell_m, tables().cell_m, sizeof(qp.cell_m));
  std::memcpy(qp.cell_below, tables().cell_below, sizeof(qp.cell_below));
  qp.dq = q->dq_group == kGroup ? 1 : 0;
  qp.dqc = qp.dq ? q->dq_code : 0;
  const int64_t groups = cdiv(nb, kGroup);
  if (groups > 0x7FFFFFFF) return QLORA_ERR_SHAPE;
  k_quantize_nf4<<<static_cast<unsigned>(groups), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(w_bf16), nb, reinterpret_cast<uint32_t*>(q->codes), q->scale_codes,
      q->absmax, qp);
  return launch_status();
}

qlora_status_t qlora_dequantize(const qlora_nf4_t* q, void* w_bf16_out, void* stream) {
  qlora_status_t s = check_nf4(q);
  if (s != QLORA_OK) return s;
  if (w_bf16_out == nullptr) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(w_bf16_out)) return QLORA_ERR_ALIGNMENT;
  int sms = 0;
  if ((s = device_ready(&sms)) != QLORA_OK) return s;
  const int64_t nwords = q->n_out * q->k_in / 8;
  DequantParams dp{};
  std::memcpy(dp.cb, tables().cb, sizeof(dp.cb));
  dp.dq = q->dq_group == kGroup ? 1 : 0;
  dp.dqc = dp.dq ? q->dq_code : 0;
  const int blocks = static_cast<int>(std::min<int64_t>(cdiv(nwords, 256), int64_t(sms) * 16));
  k_dequantize_nf4<<<std::max(blocks, 1), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const uint32_t*>(q->codes), q->scale_codes, q->absmax, nwords,
      static_cast<uint4*>(w_bf16_out), dp);
  return launch_status();
}

qlora_status_t qlora_linear_fwd_ex(const qlora_nf4_t* q, const void* x, int64_t m, const void* a,
                                   const void* b, int32_t r, float alpha, void* y, void* u_out,
                                   void* ws, size_t ws_bytes, int32_t path, void* stream) {
  int sms = 0, pairs = 0;
  qlora_status_t s = check_nf4(q);
  if (s != QLORA_OK) return s;
  if (path < QLORA_FWD_AUTO || path > QLORA_FWD_GEMV) return QLORA_ERR_INVALID_ARG;
  if ((s = device_ready(&sms, &pairs)) != QLORA_OK) return s;
  const LinearArgs la{q, m, r, alpha, ws, ws_bytes};
  if ((s = check_linear(la, sms, true)) != QLORA_OK) return s;
  if (m == 0) return QLORA_OK;
  if (x == nullptr || a == nullptr || b == nullptr || y == nullptr) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(a) || !aligned16(b) || !aligned16(y) || (u_out && !aligned16(u_out)))
    return QLORA_ERR_ALIGNMENT;
  if (path == QLORA_FWD_AUTO) path = (m <= kGemvMaxM) ? QLORA_FWD_GEMV : QLORA_FWD_GEMM;
  if (path == QLORA_FWD_GEMV && m > kGemvMaxM) return QLORA_ERR_SHAPE;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t n = q->n_out, k = q->k_in;
  const int32_t r64 = r64_of(r);
  const float sc = alpha / static_cast<float>(r);
  const int mode = g_sched.load();
  const WsPlan wp = plan_ws(m, n, k, r, sms, true, mode);
  uint8_t* wsb = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  __nv_bfloat16* u_pad = reinterpret_cast<__nv_bfloat16*>(wsb);
  __nv_bfloat16* b_pad = reinterpret_cast<__nv_bfloat16*>(wsb + wp.u_pad + wp.v_pad);
  float* part = reinterpret_cast<float*>(wsb + wp.u_pad + wp.v_pad + wp.b_pad + wp.dy_pad);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const auto* ab = static_cast<const __nv_bfloat16*>(a);
  const auto* bb = static_cast<const __nv_bfloat16*>(b);
  const __nv_bfloat16* b_use = bb;
  int64_t ldb = r;
  // stream-K flags, zeroed before the call's first kernel (the chain of
  // kernels below runs as programmatic dependents, with no memset between)
  uint32_t* sk_flags = nullptr;
  if (path == QLORA_FWD_GEMM && wp.sk_ok && ws_bytes >= wp.sk_total) {
    sk_flags = reinterpret_cast<uint32_t*>(wsb + wp.flags_off);
    if (cudaMemsetAsync(sk_flags, 0, sk_flag_bytes(sms), st) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
  }
  if (r % 8 != 0) {
    if ((s = pad_cols(bb, b_pad, n, r, r64, sms, st)) != QLORA_OK) return s;
    b_use = b_pad;
    ldb = r64;
  }

  if (path == QLORA_FWD_GEMV) {
    LoraDownSmallParams lp{};
    lp.x = xb;
    lp.a = ab;
    lp.u_pad = u_pad;
    lp.u_out = static_cast<__nv_bfloat16*>(u_out);
    lp.k = k;
    lp.m = static_cast<int32_t>(m);
    lp.r = r;
    lp.r64 = r64;
    lp.s = sc;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t dcfg = {};
    // m = 1: 16 CTAs of 16 warps, four ranks per CTA per pass; else one CTA of 4 warps per rank
    dcfg.gridDim = dim3(static_cast<unsigned>(m == 1 ? std::min<int64_t>(16, cdiv(r64, 4)) : r64), 1, 1);
    dcfg.blockDim = dim3(m == 1 ? 512 : 128, 1, 1);
    dcfg.stream = st;
    dcfg.attrs = attr;
    dcfg.numAttrs = 1;
    const cudaError_t de = (m == 1)   ? cudaLaunchKernelEx(&dcfg, k_lora_down_small<1>, lp)
                           : (m <= 8) ? cudaLaunchKernelEx(&dcfg, k_lora_down_small<8>, lp)
                                      : cudaLaunchKernelEx(&dcfg, k_lora_down_small<16>, lp);
    if (de != cudaSuccess) {
      g_launches.fetch_add(1, std::memory_order_relaxed);
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    if ((s = launch_status()) != QLORA_OK) return s;
    GemvParams gp{};
    gp.codes = q->codes;
    gp.q2 = q->scale_codes;
    gp.smax = q->absmax;
    gp.x = xb;
    gp.u = u_pad;
    gp.b = b_use;
    gp.y = static_cast<__nv_bfloat16*>(y);
    gp.n = n;
    gp.k = k;
    gp.m = static_cast<int32_t>(m);
    gp.r = r;
    gp.r64 = r64;
    gp.ldb = static_cast<int32_t>(ldb);
    std::memcpy(gp.cb, tables().cb, sizeof(gp.cb));
    gp.dq = q->dq_group == kGroup ? 1 : 0;
    gp.dqc = gp.dq ? q->dq_code : 0;
    // launched as a programmatic dependent of the x A^T kernel: its weight
    // stream starts while u' is still being computed
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cdiv(n, 16)), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // one instantiation per token-group count and block-scale format
    using GemvKernel = void (*)(GemvParams);
    static constexpr GemvKernel kGemv[2][4] = {
        {k_gemv_nf4<1, kScNone>, k_gemv_nf4<1, kScU8x256>, k_gemv_nf4<1, kScU8x255>, k_gemv_nf4<1, kScS8Mid>},
        {k_gemv_nf4<2, kScNone>, k_gemv_nf4<2, kScU8x256>, k_gemv_nf4<2, kScU8x255>, k_gemv_nf4<2, kScS8Mid>}};
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kGemv[m <= 8 ? 0 : 1][scale_format(gp.dq, gp.dqc)], gp);
    if (e != cudaSuccess) {
      g_launches.fetch_add(1, std::memory_order_relaxed);
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
    return launch_status();
  }

  // u' = bf16(s x A^T) through the tensor cores (split over K)
  CUtensorMap m_x_a, m_at, m_x_b, m_u, m_codes;
  if (!map_bf16(&m_x_a, xb, m, k, k, 128) || !map_bf16(&m_at, ab, r, k, k, static_cast<uint32_t>(r64)))
    return QLORA_ERR_CUDA;
  s = lora_product<A_TMA_K, B_TMA_K>(m_x_a, m_at, m, k, r, sc, 0, u_pad, static_cast<__nv_bfloat16*>(u_out),
                                     nullptr, part, sms, st);
  if (s != QLORA_OK) return s;

  // y^T tiles: A = restored W (on chip), B = x, plus u' B^T as extra k-tiles
  if (!map_bf16(&m_x_b, xb, m, k, k, 128) || !map_bf16(&m_u, u_pad, m, r64, r64, 128) ||
      !map2d(&m_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, q->codes, static_cast<uint64_t>(k / 2),
             static_cast<uint64_t>(n), static_cast<uint64_t>(k / 2), 32, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
    return QLORA_ERR_CUDA;
  TcParams p{};
  p.rows = static_cast<int32_t>(n);
  p.cols = static_cast<int32_t>(m);
  p.kt_main = static_cast<int32_t>(k / 64);
  p.kt_lora = r64 / 64;
  p.kt_split = p.kt_main;
  p.tiles_rows = static_cast<int32_t>(cdiv(n, 256));
  p.tiles_cols = static_cast<int32_t>(cdiv(m, 256));
  p.splits = 1;
  p.q2 = q->scale_codes;
  p.smax = q->absmax;
  p.kblocks = k / 64;
  p.nblocks = n * (k / 64);
  p.dq = q->dq_group == kGroup ? 1 : 0;
  p.dqc = p.dq ? q->dq_code : 0;
  p.w_rows = n;
  p.w_cols = k;
  std::memcpy(p.cb, tables().cb, sizeof(p.cb));
  p.lora = b_use;
  p.lora_ld = ldb;
  p.lora_r = (r % 8 != 0) ? r64 : r;
  p.out = y;
  p.ldo = n;
  return launch_pair<A_DQ_K>(pairs, m, st, m_x_b, m_u, m_codes, p,
                             sk_flags != nullptr ? reinterpret_cast<uint8_t*>(part) : nullptr, sk_flags, sms, mode);
}

qlora_status_t qlora_linear_fwd(const qlora_nf4_t* q, const void* x, int64_t m, const void* a, const void* b,
                                int32_t r, float alpha, void* y, void* u_out, void* ws, size_t ws_bytes,
                                void* stream) {
  return qlora_linear_fwd_ex(q, x, m, a, b, r, alpha, y, u_out, ws, ws_bytes, QLORA_FWD_AUTO, stream);
}

qlora_status_t qlora_linear_bwd(const qlora_nf4_t* q, const void* x, const void* u, const void* dy, int64_t m,
                                const void* a, const void* b, int32_t r, float alpha, void* dx, float* da,
                                float* db, void* ws, size_t ws_bytes, void* stream) {
  int sms = 0, pairs = 0;
  qlora_status_t s = check_nf4(q);
  if (s != QLORA_OK) return s;
  if ((s = device_ready(&sms, &pairs)) != QLORA_OK) return s;
  const LinearArgs la{q, m, r, alpha, ws, ws_bytes};
  if ((s = check_linear(la, sms, false)) != QLORA_OK) return s;
  if (da == nullptr || db == nullptr) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(da) || !aligned16(db)) return QLORA_ERR_ALIGNMENT;
  const int64_t n = q->n_out, k = q->k_in;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (m == 0) {
    // no tokens (x, u, dY, A, B and dX are not read): the gradients are exactly zero
    if (cudaMemsetAsync(da, 0, static_cast<size_t>(r) * k * sizeof(float), st) != cudaSuccess ||
        cudaMemsetAsync(db, 0, static_cast<size_t>(n) * r * sizeof(float), st) != cudaSuccess)
      return QLORA_ERR_CUDA;
    return QLORA_OK;
  }
  if (x == nullptr || dy == nullptr || a == nullptr || b == nullptr) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(dy) || !aligned16(a) || !aligned16(b) || (dx && !aligned16(dx)) ||
      (u && !aligned16(u)))
    return QLORA_ERR_ALIGNMENT;
  const int32_t r64 = r64_of(r);
  const float sc = alpha / static_cast<float>(r);
  const int mode = g_sched.load();
  const WsPlan wp = plan_ws(m, n, k, r, sms, false, mode);
  uint8_t* wsb = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  __nv_bfloat16* u_pad = reinterpret_cast<__nv_bfloat16*>(wsb);
  __nv_bfloat16* v_pad = reinterpret_cast<__nv_bfloat16*>(wsb + wp.u_pad);
  __nv_bfloat16* b_pad = reinterpret_cast<__nv_bfloat16*>(wsb + wp.u_pad + wp.v_pad);
  __nv_bfloat16* dy_pad = reinterpret_cast<__nv_bfloat16*>(wsb + wp.u_pad + wp.v_pad + wp.b_pad);
  float* part = reinterpret_cast<float*>(wsb + wp.u_pad + wp.v_pad + wp.b_pad + wp.dy_pad);
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const auto* ab = static_cast<const __nv_bfloat16*>(a);
  const auto* bb = static_cast<const __nv_bfloat16*>(b);
  const auto* dyb = static_cast<const __nv_bfloat16*>(dy);
  // stream-K flags, zeroed before the call's first kernel (the chain of
  // kernels below runs as programmatic dependents, with no memset between)
  uint32_t* sk_flags = nullptr;
  if (dx != nullptr && wp.sk_ok && ws_bytes >= wp.sk_total) {
    sk_flags = reinterpret_cast<uint32_t*>(wsb + wp.flags_off);
    if (cudaMemsetAsync(sk_flags, 0, sk_flag_bytes(sms), st) != cudaSuccess) {
      cudaGetLastError();
      return QLORA_ERR_CUDA;
    }
  }
  // dY rows reach the tensor maps with a 16-byte stride: pad them when N % 8 != 0
  const int64_t ldn = rup(n, 8);
  if (ldn != n) {
    if ((s = pad_cols(dyb, dy_pad, m, static_cast<int32_t>(n), static_cast<int32_t>(ldn), sms, st)) != QLORA_OK)
      return s;
    dyb = dy_pad;
  }
  const __nv_bfloat16* b_use = bb;
  int64_t ldb = r;
  if (r % 8 != 0) {
    if ((s = pad_cols(bb, b_pad, n, r, r64, sms, st)) != QLORA_OK) return s;
    b_use = b_pad;
    ldb = r64;
  }

  // u' (saved by the forward, padded here when needed, or recomputed)
  const __nv_bfloat16* u_use = nullptr;
  int64_t ldu = r64;
  if (u != nullptr && r % 8 == 0) {
    u_use = static_cast<const __nv_bfloat16*>(u);
    ldu = r;
  } else if (u != nullptr) {
    if ((s = pad_cols(static_cast<const __nv_bfloat16*>(u), u_pad, m, r, r64, sms, st)) != QLORA_OK) return s;
    u_use = u_pad;
  } else {
    CUtensorMap m_x_a, m_at;
    if (!map_bf16(&m_x_a, xb, m, k, k, 128) || !map_bf16(&m_at, ab, r, k, k, static_cast<uint32_t>(r64)))
      return QLORA_ERR_CUDA;
    s = lora_product<A_TMA_K, B_TMA_K>(m_x_a, m_at, m, k, r, sc, 0, u_pad, nullptr, nullptr, part, sms, st);
    if (s != QLORA_OK) return s;
    u_use = u_pad;
  }

  // v' = bf16(s dY B): A = dY (K-major), B = B_lora seen MN-major, reduction over N
  {
    CUtensorMap m_dy_a, m_bmn;
    if (!map_bf16(&m_dy_a, dyb, m, n, ldn, 128) || !map_bf16(&m_bmn, b_use, n, ldb == r ? r : r64, ldb, 64))
      return QLORA_ERR_CUDA;
    s = lora_product<A_TMA_K, B_TMA_MN>(m_dy_a, m_bmn, m, n, r, sc, 0, v_pad, nullptr, nullptr, part, sms, st);
    if (s != QLORA_OK) return s;
  }

  // dB [N x r] = dY^T u'  (A = dY seen MN-major, B = u' MN-major), right after
  // dY B so that much of dY is still in L2 when it is read again
  {
    CUtensorMap m_dymn, m_umn;
    if (!map_bf16(&m_dymn, dyb, m, n, ldn, 64) || !map_bf16(&m_umn, u_use, m, ldu == r ? r : r64, ldu, 64))
      return QLORA_ERR_CUDA;
    s = lora_product<A_TMA_MN, B_TMA_MN>(m_dymn, m_umn, n, m, r, 1.0f, 1, nullptr, nullptr, db, part, sms, st);
    if (s != QLORA_OK) return s;
  }
  // dX^T tiles: A = restored W seen MN-major (reduction over d_out), B = dY,
  // plus v' A_lora as extra k-tiles
  if (dx != nullptr) {
    CUtensorMap m_dy_b, m_v, m_codes;
    if (!map_bf16(&m_dy_b, dyb, m, n, ldn, 128) || !map_bf16(&m_v, v_pad, m, r64, r64, 128) ||
        !map2d(&m_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, q->codes, static_cast<uint64_t>(k / 2),
               static_cast<uint64_t>(n), static_cast<uint64_t>(k / 2), 64, 64, CU_TENSOR_MAP_SWIZZLE_NONE))
      return QLORA_ERR_CUDA;
    TcParams p{};
    p.rows = static_cast<int32_t>(k);
    p.cols = static_cast<int32_t>(m);
    p.kt_main = static_cast<int32_t>(cdiv(n, 64));
    p.kt_lora = r64 / 64;
    p.kt_split = p.kt_main;
    p.tiles_rows = static_cast<int32_t>(cdiv(k, 256));
    p.tiles_cols = static_cast<int32_t>(cdiv(m, 256));
    p.splits = 1;
    p.q2 = q->scale_codes;
    p.smax = q->absmax;
    p.kblocks = k / 64;
    p.nblocks = n * (k / 64);
    p.dq = q->dq_group == kGroup ? 1 : 0;
    p.dqc = p.dq ? q->dq_code : 0;
    p.w_rows = n;
    p.w_cols = k;
    std::memcpy(p.cb, tables().cb, sizeof(p.cb));
    p.lora = ab;
    p.lora_ld = k;
    p.lora_r = r;
    p.out = dx;
    p.ldo = k;
    s = launch_pair<A_DQ_MN>(pairs, m, st, m_dy_b, m_v, m_codes, p,
                             sk_flags != nullptr ? reinterpret_cast<uint8_t*>(part) : nullptr, sk_flags, sms, mode);
    if (s != QLORA_OK) return s;
  }

  // dA^T [K x r] = x^T v'  (A = x seen MN-major, B = v' MN-major, reduction over tokens)
  {
    CUtensorMap m_xmn, m_vmn;
    if (!map_bf16(&m_xmn, xb, m, k, k, 64) || !map_bf16(&m_vmn, v_pad, m, r64, r64, 64)) return QLORA_ERR_CUDA;
    s = lora_product<A_TMA_MN, B_TMA_MN>(m_xmn, m_vmn, k, m, r, 1.0f, 2, nullptr, nullptr, da, part, sms, st);
    if (s != QLORA_OK) return s;
  }
  return QLORA_OK;
}

qlora_status_t qlora_merge_lora(const qlora_nf4_t* q, const void* a, const void* b, int32_t r, float alpha,
                                void* w_out, void* stream) {
  qlora_status_t s = check_nf4(q);
  if (s != QLORA_OK) return s;
  if (r < 1 || r > kMaxRank) return QLORA_ERR_SHAPE;
  if (!std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
  if (a == nullptr || b == nullptr || w_out == nullptr) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(w_out)) return QLORA_ERR_ALIGNMENT;
  // B is read 16 bytes at a time when r % 8 == 0, else element by element
  if ((reinterpret_cast<uintptr_t>(b) & ((r % 8 == 0) ? 15u : 1u)) != 0) return QLORA_ERR_ALIGNMENT;
  int sms = 0;
  if ((s = device_ready(&sms)) != QLORA_OK) return s;
  MergeParams p{};
  p.codes = q->codes;
  p.q2 = q->scale_codes;
  p.smax = q->absmax;
  p.a = static_cast<const __nv_bfloat16*>(a);
  p.b = static_cast<const __nv_bfloat16*>(b);
  p.out = static_cast<__nv_bfloat16*>(w_out);
  p.n = q->n_out;
  p.k = q->k_in;
  p.r = r;
  p.r64 = r64_of(r);
  p.s = alpha / static_cast<float>(r);
  std::memcpy(p.cb, tables().cb, sizeof(p.cb));
  p.dq = q->dq_group == kGroup ? 1 : 0;
  p.dqc = p.dq ? q->dq_code : 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the tensor-core merge takes B through TMA (16-byte rows: r % 8 == 0)
  if (r % 8 == 0) {
    CUtensorMap m_b, m_a, m_codes, m_out;
    if (!map_bf16(&m_b, b, p.n, r, r, 128) || !map_bf16(&m_a, a, r, p.k, p.k, 64) ||
        !map2d(&m_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, q->codes, static_cast<uint64_t>(p.k / 2),
               static_cast<uint64_t>(p.n), static_cast<uint64_t>(p.k / 2), 128, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !map2d(&m_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w_out, static_cast<uint64_t>(p.k), static_cast<uint64_t>(p.n),
               static_cast<uint64_t>(p.k) * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
      return QLORA_ERR_CUDA;
    p.tiles_n = static_cast<int32_t>(cdiv(p.n, 128));
    p.tiles_k = static_cast<int32_t>(cdiv(p.k, 256));
    const int64_t tiles = static_cast<int64_t>(p.tiles_n) * p.tiles_k;
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(tiles, sms));
    k_merge_tc<<<grid, 32 * (2 + kMergeDrainWarps), merge_tc_smem_bytes(), st>>>(m_b, m_a, m_codes, m_out, p);
    return launch_status();
  }
  const size_t smem = merge_smem_bytes(p.r64);
  const dim3 grid(static_cast<unsigned>(cdiv(p.k, 128)), static_cast<unsigned>(cdiv(p.n, 128)), 1);
  if (grid.y > 65535u) return QLORA_ERR_SHAPE;
  k_merge_lora<<<grid, 256, smem, st>>>(p);
  return launch_status();
}

namespace {
// Argument checks of the AdamW entry points (nothing enqueued yet).
qlora_status_t check_adamw(const float* master, const void* param_bf16, const float* grad, const float* m,
                           const float* v, int64_t n, const qlora_adamw_t* hp) {
  if (hp == nullptr || n < 0) return QLORA_ERR_INVALID_ARG;
  if (n == 0) return QLORA_OK;
  if (master == nullptr || grad == nullptr || m == nullptr || v == nullptr) return QLORA_ERR_INVALID_ARG;
  if (hp->step < 1 || !(hp->lr >= 0.0f) || !(hp->beta1 >= 0.0f && hp->beta1 < 1.0f) ||
      !(hp->beta2 >= 0.0f && hp->beta2 < 1.0f) || !(hp->eps > 0.0f) || !std::isfinite(hp->weight_decay))
    return QLORA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(master) | reinterpret_cast<uintptr_t>(grad) | reinterpret_cast<uintptr_t>(m) |
       reinterpret_cast<uintptr_t>(v)) & 3u)
    return QLORA_ERR_ALIGNMENT;
  if (param_bf16 != nullptr && (reinterpret_cast<uintptr_t>(param_bf16) & 1u)) return QLORA_ERR_ALIGNMENT;
  return QLORA_OK;
}
}  // namespace

qlora_status_t qlora_adamw_staged(float* master, void* param_bf16, const float* grad, float* m_host, float* v_host,
                                  float* m_stage, float* v_stage, int64_t n, const qlora_adamw_t* hp, void* stream) {
  qlora_status_t s = check_adamw(master, param_bf16, grad, m_stage, v_stage, n, hp);
  if (s != QLORA_OK || n == 0) return s;
  if (m_host == nullptr || v_host == nullptr) return QLORA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(m_host) | reinterpret_cast<uintptr_t>(v_host)) & 3u) return QLORA_ERR_ALIGNMENT;
  if ((s = device_ready(nullptr)) != QLORA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(n) * sizeof(float);
  if (cudaMemcpyAsync(m_stage, m_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
      cudaMemcpyAsync(v_stage, v_host, bytes, cudaMemcpyHostToDevice, st) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  if ((s = qlora_adamw_step(master, param_bf16, grad, m_stage, v_stage, n, hp, stream)) != QLORA_OK) return s;
  if (cudaMemcpyAsync(m_host, m_stage, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemcpyAsync(v_host, v_stage, bytes, cudaMemcpyDeviceToHost, st) != cudaSuccess) {
    cudaGetLastError();
    return QLORA_ERR_CUDA;
  }
  return QLORA_OK;
}

qlora_status_t qlora_adamw_step(float* master, void* param_bf16, const float* grad, float* m, float* v, int64_t n,
                                const qlora_adamw_t* hp, void* stream) {
  qlora_status_t s = check_adamw(master, param_bf16, grad, m, v, n, hp);
  if (s != QLORA_OK || n == 0) return s;
  const auto a4 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  int sms = 0;
  if ((s = device_ready(&sms)) != QLORA_OK) return s;
  AdamwParams a{};
  a.master = master;
  a.grad = grad;
  a.m = m;
  a.v = v;
  a.param = static_cast<__nv_bfloat16*>(param_bf16);
  a.n = n;
  a.beta1 = hp->beta1;
  a.beta2 = hp->beta2;
  a.eps = hp->eps;
  // step constants in double, rounded once
  const double bc1 = 1.0 - std::pow(static_cast<double>(hp->beta1), hp->step);
  const double bc2 = 1.0 - std::pow(static_cast<double>(hp->beta2), hp->step);
  a.decay = static_cast<float>(1.0 - static_cast<double>(hp->lr) * hp->weight_decay);
  a.step_size = static_cast<float>(hp->lr / bc1);
  a.inv_sqrt_bc2 = static_cast<float>(1.0 / std::sqrt(bc2));
  a.vec4 = a4(master) && a4(grad) && a4(m) && a4(v) &&
           (param_bf16 == nullptr || (reinterpret_cast<uintptr_t>(param_bf16) & 7u) == 0);
  const int blocks = static_cast<int>(std::min<int64_t>(cdiv(cdiv(n, 4), 256), int64_t(sms) * 8));
  k_adamw<<<std::max(blocks, 1), 256, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return launch_status();
}

static_assert(QLORA_DEV_TIMEOUT_PRODUCER == QLORA_STATUS_BIT_PRODUCER && QLORA_DEV_TIMEOUT_MMA == QLORA_STATUS_BIT_MMA &&
                  QLORA_DEV_TIMEOUT_APROD == QLORA_STATUS_BIT_RESTORE && QLORA_DEV_TIMEOUT_EPI == QLORA_STATUS_BIT_EPILOGUE &&
                  QLORA_DEV_TIMEOUT_SELFTEST == QLORA_STATUS_BIT_SELFTEST,
              "device status bits match the header");

qlora_status_t qlora_selftest_wait_timeout(uint32_t limit_us, void* stream) {
  int sms = 0, pairs = 0;
  qlora_status_t s = device_ready(&sms, &pairs);
  if (s != QLORA_OK) return s;
  const uint64_t us = std::min<uint64_t>(std::max<uint32_t>(limit_us, 1u), 2000000u);
  k_selftest_wait<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(us * 1000ull);
  return launch_status();
}

qlora_status_t qlora_device_status(void* stream, uint32_t* bits) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QLORA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_dev_status, sizeof(v)) != cudaSuccess) return QLORA_ERR_CUDA;
  const unsigned int zero = 0;
  if (v != 0 && cudaMemcpyToSymbol(g_dev_status, &zero, sizeof(zero)) != cudaSuccess) return QLORA_ERR_CUDA;
  if (bits) *bits = v;
  return v ? QLORA_ERR_TIMEOUT : QLORA_OK;
}

}  // extern "C"
