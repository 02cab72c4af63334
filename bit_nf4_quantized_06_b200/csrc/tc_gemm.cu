// tcgen05 GEMM engine for the small LoRA products on sm_100a (x A^T, dY B,
// dA, dB): both operands come from TMA (K-major or MN-major 128-byte swizzled
// tiles), persistent CTAs (at most one per SM) walk 128 x BN output tiles,
// split along the reduction when there are fewer tiles than SMs, and two
// accumulators in tensor memory let the drain of tile i overlap the main
// loop of tile i + 1. fp32 partial tiles go to a workspace slab per split
// and a fixed-order reduction kernel finishes them (deterministic):
// bf16(s * u) for x A^T and dY B, fp32 dA (transposed) and dB. Without a
// split the drain writes those results itself and no reduction runs.
//
//   D[128 x BN] (fp32, tensor memory)  +=  A[128 x 64] * B[BN x 64]^T  per k-tile
//
// Warp roles: warp 0 issues TMA loads (one lane), warp 1 allocates tensor
// memory and issues tcgen05.mma (one lane), warps 2-5 drain the accumulator.
// Every pipeline wait is bounded (see ptx.cuh); every TMA load fills only the
// issuing CTA's shared memory.
#include "kernels.h"
#include "nf4_dev.cuh"
#include "ptx.cuh"
#include "tc_common.cuh"

namespace qlora {

using namespace tcd;

namespace {

template <int BN>
constexpr uint32_t tmem_cols() {
  return BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
}

// The last step of the split reduction for columns [c0, c0 + 32) of output
// row `row`, given their complete fp32 sums v (what k_reduce_splits does
// after summing the slabs): mode 0 bf16(scale * v) to out_pad [rows x ld]
// and out_c [rows x cols] (if set), mode 1 fp32 out_f [rows x cols], mode 2
// fp32 out_f [cols x rows] (consecutive lanes hold consecutive rows, so the
// transposed stores of a warp coalesce).
__device__ __forceinline__ void finish_row(const SmallParams& p, int row, int c0, const uint32_t (&v)[32]) {
  if (p.mode == 0) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
      pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * p.scale, __uint_as_float(v[2 * i + 1]) * p.scale);
    uint4* dst = reinterpret_cast<uint4*>(p.out_pad + static_cast<int64_t>(row) * p.ld + c0);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
    if (p.out_c != nullptr) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (c0 + i < p.cols)
          p.out_c[static_cast<int64_t>(row) * p.cols + c0 + i] = __float2bfloat16_rn(__uint_as_float(v[i]) * p.scale);
    }
  } else if (p.mode == 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (c0 + i < p.cols) p.out_f[static_cast<int64_t>(row) * p.cols + c0 + i] = __uint_as_float(v[i]) * p.scale;
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (c0 + i < p.cols) p.out_f[static_cast<int64_t>(c0 + i) * p.rows + row] = __uint_as_float(v[i]) * p.scale;
  }
}

}  // namespace

template <int BN, int AS, int BS, int STAGES>
__global__ void __launch_bounds__(192, 1)
    k_tc_small(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b, SmallParams p) {
  constexpr bool A_MN = (AS == A_TMA_MN);
  constexpr bool B_MN = (BS == B_TMA_MN);
  constexpr uint32_t A_BYTES = 16384;
  constexpr uint32_t B_BYTES = BN * 128;
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  constexpr uint32_t IDESC = idesc_bf16_f32(128, BN, A_MN, B_MN);
  constexpr uint32_t ACC_COLS = tmem_cols<BN>();
  constexpr uint32_t TMEM_ALLOC = 2 * ACC_COLS;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(TMEM_ALLOC <= 512, "tensor memory");

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const ctl = smem_raw + (base - raw) + STAGES * STAGE_BYTES;
  const uint32_t bar0 = base + STAGES * STAGE_BYTES;
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto bar_accf = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto bar_acce = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 + b); };
  const uint32_t bar_fin = bar0 + 8u * (2 * STAGES + 4);
  uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(ctl + 8 * (2 * STAGES + 5));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(ctl + 8 * (2 * STAGES + 5) + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntile_total = p.tiles * p.splits;
  // tile index = row tile * splits + split
  auto row0_of = [&](int tile) { return (tile / p.splits) * 128; };
  auto kbeg_of = [&](int tile) { return (tile % p.splits) * p.kt_split; };
  auto nk_of = [&](int tile) {
    const int kb = kbeg_of(tile);
    return max(0, min(p.kt_main, kb + p.kt_split) - kb);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf(b), 1);
      mbar_init(bar_acce(b), 4);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_ALLOC);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // launched as a programmatic dependent: the set-up above overlapped the
  // kernel in front; its results are visible from here on
  grid_dependency_wait();
  grid_dependency_trigger();

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntile_total; tile += gridDim.x) {
        const int row0 = row0_of(tile);
        const int kb = kbeg_of(tile);
        const int nk = nk_of(tile);
        for (int t = 0; t < nk; ++t, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(bar_empty(s), ph ^ 1, abort_flag, QLORA_DEV_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          const uint32_t a_s = base + s * STAGE_BYTES;
          const uint32_t b_s = a_s + A_BYTES;
          const int kt = kb + t;
          mbar_arrive_expect_tx(bar_full(s), A_BYTES + B_BYTES);
          if (BS == B_TMA_K) {
            tma_load_2d(b_s, &tm_b, bar_full(s), kt * 64, 0);
          } else {
#pragma unroll
            for (int i = 0; i < BN / 64; ++i) tma_load_2d(b_s + i * 8192, &tm_b, bar_full(s), 64 * i, kt * 64);
          }
          if (AS == A_TMA_K) {
            tma_load_2d(a_s, &tm_a, bar_full(s), kt * 64, row0);
          } else {
            tma_load_2d(a_s, &tm_a, bar_full(s), row0, kt * 64);
            tma_load_2d(a_s + 8192, &tm_a, bar_full(s), row0 + 64, kt * 64);
          }
        }
      }
      // let every load this thread started land before the CTA can exit
      for (int j = max(0, it - STAGES); j < it; ++j) drain_wait(bar_full(j % STAGES), (j / STAGES) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntile_total; tile += gridDim.x, ++tcount) {
        const int nk = nk_of(tile);
        const int b = tcount & 1;
        const uint32_t aph = (tcount >> 1) & 1;
        if (!mbar_wait(bar_acce(b), aph ^ 1, abort_flag, QLORA_DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * ACC_COLS;
        for (int t = 0; t < nk; ++t, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(bar_full(s), ph, abort_flag, QLORA_DEV_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_s = base + s * STAGE_BYTES;
          const uint32_t b_s = a_s + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t da = A_MN ? smem_desc_sw128(a_s + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(a_s + kk * 32, 16, 1024);
            const uint64_t db = B_MN ? smem_desc_sw128(b_s + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(b_s + kk * 32, 16, 1024);
            tc_mma_ss(d_tmem, da, db, IDESC, (t > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar_empty(s));
        }
        if (ok) tc_commit(bar_accf(b));
      }
      tc_commit(bar_fin);
      drain_wait(bar_fin, 0);
    }
  } else {
    // ---------------------------------------------------------------- epilogue: fp32 partial slab
    const int quarter = warp & 3;  // TMEM lanes [32 q, 32 q + 32) belong to warp % 4
    int tcount = 0;
    for (int tile = blockIdx.x; tile < ntile_total; tile += gridDim.x, ++tcount) {
      const int b = tcount & 1;
      const uint32_t aph = (tcount >> 1) & 1;
      bool ok = mbar_wait(bar_accf(b), aph, abort_flag, QLORA_DEV_TIMEOUT_EPI);
      if (!warp_all(ok)) break;
      tc_fence_after();
      const int prow = row0_of(tile) + quarter * 32 + lane;
      const bool empty = nk_of(tile) == 0;
      const uint32_t taddr = tmem_base + b * ACC_COLS + (static_cast<uint32_t>(quarter * 32) << 16);
      float* out = p.part + (static_cast<int64_t>(tile % p.splits) * p.rows_pad + prow) * BN;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + ch * 32, r);
        tc_wait_ld();
        if (empty) {
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = 0u;
        }
        if (p.splits == 1) {
          // one split: this is the whole sum, so the reduction's final step
          // (scale, convert, layout) is done here and no slab is written
          if (prow < p.rows) finish_row(p, prow, ch * 32, r);
          continue;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
          reinterpret_cast<float4*>(out + ch * 32)[i] =
              make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]), __uint_as_float(r[4 * i + 2]),
                          __uint_as_float(r[4 * i + 3]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_acce(b));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_ALLOC);
  }
}

// Sum the split slabs in split order (deterministic) and write the result:
// mode 0: bf16(scale * sum) to out_pad [rows x ld] and out_c [rows x cols]
// (if set); mode 1: fp32 out_f [rows x cols]; mode 2: fp32 out_f [cols x rows].
// Each thread handles four consecutive columns of one row; for mode 2 rows
// run fastest across threads so that the transposed writes coalesce.
__global__ void __launch_bounds__(256) k_reduce_splits(SmallParams p) {
  grid_dependency_wait();
  grid_dependency_trigger();
  const int q4 = p.ld >> 2;
  const int total = p.rows * q4;
  const int64_t slab = static_cast<int64_t>(p.rows_pad) * p.ld;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    int row, c4;
    if (p.mode == 2) {
      row = i % p.rows;
      c4 = i / p.rows;
    } else {
      row = i / q4;
      c4 = i - row * q4;
    }
    const float* src = p.part + static_cast<int64_t>(row) * p.ld + 4 * c4;
    float4 acc = __ldcs(reinterpret_cast<const float4*>(src));
    for (int z = 1; z < p.splits; ++z) {
      const float4 v = __ldcs(reinterpret_cast<const float4*>(src + z * slab));
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    const float a[4] = {acc.x * p.scale, acc.y * p.scale, acc.z * p.scale, acc.w * p.scale};
    const int c0 = 4 * c4;
    if (p.mode == 0) {
      uint2 pk;
      pk.x = pack_bf16x2(a[0], a[1]);
      pk.y = pack_bf16x2(a[2], a[3]);
      *reinterpret_cast<uint2*>(p.out_pad + static_cast<int64_t>(row) * p.ld + c0) = pk;
      if (p.out_c != nullptr) {
#pragma unroll
        for (int t = 0; t < 4; ++t)
          if (c0 + t < p.cols) p.out_c[static_cast<int64_t>(row) * p.cols + c0 + t] = __float2bfloat16_rn(a[t]);
      }
    } else if (p.mode == 1) {
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (c0 + t < p.cols) p.out_f[static_cast<int64_t>(row) * p.cols + c0 + t] = a[t];
    } else {
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (c0 + t < p.cols) p.out_f[static_cast<int64_t>(c0 + t) * p.rows + row] = a[t];
    }
  }
}

__global__ void __launch_bounds__(256) k_pad_cols(const __nv_bfloat16* __restrict__ src,
                                                  __nv_bfloat16* __restrict__ dst, int64_t rows,
                                                  int32_t r, int32_t r64) {
  grid_dependency_wait();
  grid_dependency_trigger();
  const int64_t total = rows * r64;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += stride) {
    const int64_t row = i / r64;
    const int32_t col = static_cast<int32_t>(i - row * r64);
    dst[i] = (col < r) ? src[row * r + col] : __float2bfloat16_rn(0.0f);
  }
}

// ------------------------------------------------------------------ instantiations
#define QLORA_TC_SMALL(BN)                                                                        \
  template __global__ void k_tc_small<BN, A_TMA_K, B_TMA_K, small_stages(BN)>(                    \
      const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap, SmallParams);     \
  template __global__ void k_tc_small<BN, A_TMA_K, B_TMA_MN, small_stages(BN)>(                   \
      const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap, SmallParams);     \
  template __global__ void k_tc_small<BN, A_TMA_MN, B_TMA_MN, small_stages(BN)>(                  \
      const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap, SmallParams);
// LoRA products: x A^T (K-major B), dY B (MN-major B), dA / dB (MN-major A and B)
QLORA_TC_SMALL(64)
QLORA_TC_SMALL(128)
QLORA_TC_SMALL(192)
QLORA_TC_SMALL(256)

}  // namespace qlora
