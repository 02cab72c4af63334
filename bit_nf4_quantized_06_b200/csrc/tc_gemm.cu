// Generic tcgen05 GEMM engine for sm_100a: persistent CTAs (at most one per
// SM) walking 128 x BN output tiles, with two accumulators in tensor memory so
// that draining tile i overlaps the main loop of tile i + 1.
//
//   D[128 x BN] (fp32, tensor memory)  +=  A[128 x 64] * B[BN x 64]^T  per k-tile
//
// Warp roles:
//   warp 0     one lane issues TMA loads (B tiles, A tiles when A comes from
//              memory, packed NF4 code tiles when A is restored on chip)
//   warp 1     allocates tensor memory; one lane issues tcgen05.mma / commit
//   warps 2-9  (restored-A variants only) A producers, two groups of four
//              taking alternate k-tiles: per stage they turn the
//              staged 4-bit codes into bf16 directly in the 128-byte swizzled
//              shared-memory layout the tensor core reads (K-major for the
//              forward, MN-major for dX); for the appended LoRA k-tiles they
//              copy the adapter rows instead. Each thread fetches its scale
//              codes and group constants kScalePrefetch k-tiles ahead with
//              cp.async into a private shared-memory ring.
//   last 4     epilogue: wait for an accumulator, tcgen05.ld it, release it,
//              write the tile out.
//
// The forward pass ("48GB GPU Fine-Tuning a 65B Model ...", § "QLoRA Puts the
// Two Methods in Different Places": each block of W is restored to bf16,
// multiplied with the input, and the LoRA branch is added) runs with
// D = y^T tile: rows are output features, columns are tokens, A = restored W,
// B = x, and s * u' * B_lora^T appended as extra k-tiles of the same
// accumulator. dX uses D = dX^T tile with A = restored W seen MN-major (the
// 4-bit blocks run along d_in, the reduction runs along d_out) and B = dY,
// plus s * v' * A_lora as extra k-tiles. The small LoRA products (x A^T,
// dY B, dA, dB) reuse the same kernel with both operands from TMA.
//
// Every pipeline wait is bounded (see ptx.cuh); every TMA load fills only
// the issuing CTA's shared memory.
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

struct TileCoord {
  int row0, col0, z, kt_begin, nmain;
};

__device__ __forceinline__ TileCoord decode_tile(const TcParams& p, int tile) {
  TileCoord c;
  c.z = tile % p.splits;
  const int rc = tile / p.splits;
  c.col0 = (rc % p.tiles_cols);
  c.row0 = (rc / p.tiles_cols) * 128;
  c.kt_begin = c.z * p.kt_split;
  c.nmain = max(0, min(p.kt_main, c.kt_begin + p.kt_split) - c.kt_begin);
  return c;
}

}  // namespace

template <int BN, int AS, int BS, int EP, int STAGES>
__global__ void __launch_bounds__(tc_threads<AS>(), 1)
    k_tc_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
              const __grid_constant__ CUtensorMap tm_b_lora,
              const __grid_constant__ CUtensorMap tm_codes, TcParams p) {
  constexpr bool DQ = tc_dq<AS>();
  constexpr bool A_MN = (AS == A_TMA_MN || AS == A_DQ_MN);
  constexpr bool B_MN = (BS == B_TMA_MN);
  constexpr uint32_t A_BYTES = 16384;
  constexpr uint32_t B_BYTES = BN * 128;
  constexpr uint32_t C_BYTES = DQ ? 4096 : 0;
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + C_BYTES;
  constexpr uint32_t IDESC = idesc_bf16_f32(128, BN, A_MN, B_MN);
  constexpr uint32_t ACC_COLS = tmem_cols<BN>();
  constexpr uint32_t TMEM_ALLOC = 2 * ACC_COLS;
  constexpr int PD = kScalePrefetch;
  constexpr int EPI_W0 = DQ ? 10 : 2;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
  static_assert(TMEM_ALLOC <= 512, "tensor memory");

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const ctl = smem_raw + (base - raw) + STAGES * STAGE_BYTES;
  const uint32_t bar0 = base + STAGES * STAGE_BYTES;
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_codes = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto bar_afull = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  auto bar_empty = [&](int s) { return bar0 + 8u * (3 * STAGES + s); };
  auto bar_accf = [&](int b) { return bar0 + 8u * (4 * STAGES + b); };
  auto bar_acce = [&](int b) { return bar0 + 8u * (4 * STAGES + 2 + b); };
  const uint32_t bar_fin = bar0 + 8u * (4 * STAGES + 4);
  uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(ctl + 8 * (4 * STAGES + 5));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(ctl + 8 * (4 * STAGES + 5) + 4);
  const uint32_t ring = bar0 + 256;  // scale-code prefetch rings, one per A-producer group

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntile_total = p.tiles_rows * p.tiles_cols * p.splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_codes(s), 1);
      mbar_init(bar_afull(s), 4);
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

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_b);
      if (!DQ) tma_prefetch_desc(&tm_a);
      if (DQ) tma_prefetch_desc(&tm_codes);
      if (p.kt_lora > 0) tma_prefetch_desc(&tm_b_lora);
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntile_total; tile += gridDim.x) {
        const TileCoord tc = decode_tile(p, tile);
        const int row0 = tc.row0;
        const int col0 = tc.col0 * BN;
        const int ntiles = tc.nmain + p.kt_lora;
        for (int t = 0; t < ntiles; ++t, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(bar_empty(s), ph ^ 1, abort_flag, QLORA_DEV_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          const uint32_t a_s = base + s * STAGE_BYTES;
          const uint32_t b_s = a_s + A_BYTES;
          const uint32_t c_s = b_s + B_BYTES;
          if (t < tc.nmain) {
            const int kt = tc.kt_begin + t;
            mbar_arrive_expect_tx(bar_full(s), B_BYTES + (DQ ? 0u : A_BYTES));
            if (BS == B_TMA_K) {
              tma_load_2d(b_s, &tm_b, bar_full(s), kt * 64, col0);
            } else {
#pragma unroll
              for (int i = 0; i < BN / 64; ++i)
                tma_load_2d(b_s + i * 8192, &tm_b, bar_full(s), col0 + 64 * i, kt * 64);
            }
            if (AS == A_TMA_K) {
              tma_load_2d(a_s, &tm_a, bar_full(s), kt * 64, row0);
            } else if (AS == A_TMA_MN) {
              tma_load_2d(a_s, &tm_a, bar_full(s), row0, kt * 64);
              tma_load_2d(a_s + 8192, &tm_a, bar_full(s), row0 + 64, kt * 64);
            } else if (AS == A_DQ_K) {
              mbar_arrive_expect_tx(bar_codes(s), C_BYTES);
              tma_load_2d(c_s, &tm_codes, bar_codes(s), kt * 32, row0);
            } else {
              mbar_arrive_expect_tx(bar_codes(s), C_BYTES);
              tma_load_2d(c_s, &tm_codes, bar_codes(s), row0 / 2, kt * 64);
            }
          } else {
            const int lt = t - tc.nmain;
            mbar_arrive_expect_tx(bar_full(s), B_BYTES);
            tma_load_2d(b_s, &tm_b_lora, bar_full(s), lt * 64, col0);
            if (DQ) mbar_arrive(bar_codes(s));  // keeps the code barrier's phase in step
          }
        }
      }
      // let every load this thread started land before the CTA can exit
      for (int j = max(0, it - STAGES); j < it; ++j) {
        drain_wait(bar_full(j % STAGES), (j / STAGES) & 1);
        if (DQ) drain_wait(bar_codes(j % STAGES), (j / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int it = 0, tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntile_total; tile += gridDim.x, ++tcount) {
        const TileCoord tc = decode_tile(p, tile);
        const int ntiles = tc.nmain + p.kt_lora;
        const int b = tcount & 1;
        const uint32_t aph = (tcount >> 1) & 1;
        if (!mbar_wait(bar_acce(b), aph ^ 1, abort_flag, QLORA_DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * ACC_COLS;
        for (int t = 0; t < ntiles; ++t, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(bar_full(s), ph, abort_flag, QLORA_DEV_TIMEOUT_MMA) ||
              (DQ && !mbar_wait(bar_afull(s), ph, abort_flag, QLORA_DEV_TIMEOUT_MMA))) {
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
  } else if (DQ && warp < EPI_W0) {
    // ---------------------------------------------------------------- A producers
    // Two groups of four warps take alternate k-tiles, so every scheduler
    // has two restore warps to switch between while one waits.
    const int grp = (warp - 2) >> 2;      // 0: warps 2-5, 1: warps 6-9
    const int tid = threadIdx.x - 64 - 128 * grp;  // 0..127 within the group
    const int ipt = p.kt_main + p.kt_lora;  // items per tile (no splits with a restored A)
    const int my_tiles = (ntile_total - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                         static_cast<int>(gridDim.x);
    const int items = my_tiles * ipt;
    const uint32_t slot0 = ring + grp * (PD * 128 * 8) + tid * 8;

    // cursor over this group's items j = grp, grp + 2, ...: k-tile t within
    // tile `tile`, whose first D row is row0
    struct Cursor {
      int j, t, tile, row0;
    };
    auto advance = [&](Cursor& c) {
      c.j += 2;
      c.t += 2;
      while (c.t >= ipt) {
        c.t -= ipt;
        c.tile += gridDim.x;
        c.row0 = (c.tile / p.tiles_cols) * 128;
      }
    };
    // this thread's weight block for k-tile t of a tile at row0 (-1 = padding)
    auto block_of = [&](int row0, int t) -> int64_t {
      if (AS == A_DQ_K) {
        const int64_t n = row0 + tid;
        return (n < p.w_rows) ? n * p.kblocks + t : -1;
      } else {
        const int64_t n = static_cast<int64_t>(t) * 64 + (tid >> 1);
        const int64_t kcol = row0 + 64 * (tid & 1);
        return (n < p.w_rows && kcol < p.w_cols) ? n * p.kblocks + (kcol >> 6) : -1;
      }
    };
    auto issue = [&](const Cursor& c, int k) {
      // prefetch ring slot k (0..PD-1) for the item under cursor c
      if (c.j < items && c.t < p.kt_main) {
        const int64_t bi = block_of(c.row0, c.t);
        const uint32_t slot = slot0 + k * (128 * 8);
        if (bi >= 0) {
          const int64_t w4 = bi & ~int64_t(3);
          const int64_t left = p.nblocks - w4;
          cp_async4(slot, p.q2 + w4, static_cast<uint32_t>(left < 4 ? left : 4));
          cp_async4(slot + 4, p.smax + (bi >> 8), 4);
        } else {
          cp_async4(slot, p.q2, 0);
          cp_async4(slot + 4, p.smax, 0);
        }
      }
      cp_async_commit();
    };

    Cursor cur{grp, grp, static_cast<int>(blockIdx.x), 0};
    cur.row0 = (cur.tile / p.tiles_cols) * 128;
    while (cur.t >= ipt) {  // only if a tile had a single item
      cur.t -= ipt;
      cur.tile += gridDim.x;
      cur.row0 = (cur.tile / p.tiles_cols) * 128;
    }
    Cursor pre = cur;
#pragma unroll 1
    for (int k = 0; k < PD - 1; ++k) {
      issue(pre, k);
      advance(pre);
    }
    int slot_use = 0, slot_issue = PD - 1;

#pragma unroll 1
    for (; cur.j < items; advance(cur)) {
      issue(pre, slot_issue);
      advance(pre);
      slot_issue = (slot_issue + 1 == PD) ? 0 : slot_issue + 1;
      const int j = cur.j;
      const int s = j % STAGES;
      const uint32_t ph = (j / STAGES) & 1;
      const int t = cur.t;
      const int row0 = cur.row0;
      const uint32_t a_s = base + s * STAGE_BYTES;
      const uint32_t c_s = a_s + A_BYTES + B_BYTES;
      bool ok = mbar_wait(bar_empty(s), ph ^ 1, abort_flag, QLORA_DEV_TIMEOUT_APROD);
      if (!warp_all(ok)) break;
      if (t < p.kt_main) {
        cp_async_wait<PD - 1>();
        const int64_t bi = block_of(row0, t);
        const uint32_t slot = slot0 + slot_use * (128 * 8);
        float sh = 0.0f;
        if (bi >= 0) {
          const uint32_t qw = lds32(slot);
          const uint32_t q2 = (qw >> (8 * static_cast<uint32_t>(bi & 3))) & 0xFFu;
          sh = restored_scale(q2, __uint_as_float(lds32(slot + 4)));
        }
        const Nf4Table tb = make_table(p.cb, sh);
        ok = mbar_wait(bar_codes(s), ph, abort_flag, QLORA_DEV_TIMEOUT_APROD);
        if (!warp_all(ok)) break;
        uint32_t src, dst, sw;
        if (AS == A_DQ_K) {
          src = c_s + tid * 32;
          dst = a_s + tid * 128;
          sw = tid & 7;
        } else {
          const int nr = tid >> 1;
          src = c_s + nr * 64 + (tid & 1) * 32;
          dst = a_s + (tid & 1) * 8192 + nr * 128;
          sw = nr & 7;
        }
        const uint4 c0 = lds128(src);
        const uint4 c1 = lds128(src + 16);
        const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          uint32_t o[4];
          lookup8(tb, words[w], o);
          sts128(dst + ((w ^ sw) << 4), o[0], o[1], o[2], o[3]);
        }
      } else {
        const int lt = t - p.kt_main;
        if (AS == A_DQ_K) {
          // forward: rows of B_lora (one output feature per thread), 64 ranks
          const int64_t n = row0 + tid;
          const uint32_t dst = a_s + tid * 128;
          const uint32_t sw = tid & 7;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4 v = make_uint4(0, 0, 0, 0);
            const int jj = lt * 64 + 8 * c;
            if (n < p.w_rows && jj < p.lora_r)
              v = __ldg(reinterpret_cast<const uint4*>(p.lora + n * p.lora_ld + jj));
            sts128(dst + ((c ^ sw) << 4), v.x, v.y, v.z, v.w);
          }
        } else {
          // dX: rows of A_lora (rank = reduction index), 64 of its d_in columns
          const int nr = tid >> 1;
          const int jr = lt * 64 + nr;
          const int64_t kcol = row0 + 64 * (tid & 1);
          const bool valid = kcol < p.w_cols && jr < p.lora_r;
          const uint32_t dst = a_s + (tid & 1) * 8192 + nr * 128;
          const uint32_t sw = nr & 7;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (valid) v = __ldg(reinterpret_cast<const uint4*>(p.lora + jr * p.lora_ld + kcol + 8 * c));
            sts128(dst + ((c ^ sw) << 4), v.x, v.y, v.z, v.w);
          }
        }
      }
      slot_use = (slot_use + 1 == PD) ? 0 : slot_use + 1;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_afull(s));
    }
    cp_async_wait<0>();
  } else if (warp >= EPI_W0) {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes [32 q, 32 q + 32) belong to warp % 4
    int tcount = 0;
    for (int tile = blockIdx.x; tile < ntile_total; tile += gridDim.x, ++tcount) {
      const TileCoord tc = decode_tile(p, tile);
      const int b = tcount & 1;
      const uint32_t aph = (tcount >> 1) & 1;
      bool ok = mbar_wait(bar_accf(b), aph, abort_flag, QLORA_DEV_TIMEOUT_EPI);
      if (!warp_all(ok)) break;
      tc_fence_after();
      const int prow = tc.row0 + quarter * 32 + lane;
      const int col0 = tc.col0 * BN;
      const uint32_t taddr = tmem_base + b * ACC_COLS + (static_cast<uint32_t>(quarter * 32) << 16);
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + ch * 32, r);
        tc_wait_ld();
        if (EP == EPI_BF16_T) {
          if (prow < p.rows) {
            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int q = col0 + ch * 32 + i;
              if (q < p.cols)
                out[static_cast<int64_t>(q) * p.ldo + prow] = __float2bfloat16_rn(__uint_as_float(r[i]));
            }
          }
        } else {
          float* out = reinterpret_cast<float*>(p.out) +
                       (static_cast<int64_t>(tc.z) * p.rows_pad + prow) * p.ldo + col0 + ch * 32;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(out)[i] =
                make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                            __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
        }
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

// ------------------------------------------------------------------ split reductions
__global__ void __launch_bounds__(256) k_reduce_splits(ReduceParams p) {
  const int64_t total = static_cast<int64_t>(p.rows) * (p.mode == 0 ? p.ld : p.cols);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t slab = static_cast<int64_t>(p.rows_pad) * p.ld;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += stride) {
    int64_t row, col;
    if (p.mode == 2) {           // transposed output: walk rows fastest
      col = i / p.rows;
      row = i - col * p.rows;
    } else {
      const int64_t w = (p.mode == 0) ? p.ld : p.cols;
      row = i / w;
      col = i - row * w;
    }
    const float* src = p.part + row * p.ld + col;
    float acc = 0.0f;
    for (int s = 0; s < p.splits; ++s) acc += src[s * slab];
    if (p.mode == 0) {
      const __nv_bfloat16 b = __float2bfloat16_rn(acc * p.scale);
      p.out_pad[row * p.ld + col] = b;
      if (p.out_c != nullptr && col < p.cols) p.out_c[row * p.cols + col] = b;
    } else if (p.mode == 1) {
      p.out_f[row * p.cols + col] = acc * p.scale;
    } else {
      p.out_f[col * p.rows + row] = acc * p.scale;
    }
  }
}

__global__ void __launch_bounds__(256) k_pad_cols(const __nv_bfloat16* __restrict__ src,
                                                  __nv_bfloat16* __restrict__ dst, int64_t rows,
                                                  int32_t r, int32_t r64) {
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
#define QLORA_TC_INST(BN, AS, BS, EP, ST)                                                        \
  template __global__ void k_tc_gemm<BN, AS, BS, EP, ST>(                                       \
      const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap,                 \
      const __grid_constant__ CUtensorMap, const __grid_constant__ CUtensorMap, TcParams);

// main forward / dX GEMMs
QLORA_TC_INST(256, A_DQ_K, B_TMA_K, EPI_BF16_T, 4)
QLORA_TC_INST(256, A_DQ_MN, B_TMA_K, EPI_BF16_T, 4)
// LoRA products: x A^T (K-major B), dY B (MN-major B), dA / dB (MN-major A and B)
#define QLORA_TC_SMALL(BN)                                  \
  QLORA_TC_INST(BN, A_TMA_K, B_TMA_K, EPI_F32_ROWS, 4)      \
  QLORA_TC_INST(BN, A_TMA_K, B_TMA_MN, EPI_F32_ROWS, 4)     \
  QLORA_TC_INST(BN, A_TMA_MN, B_TMA_MN, EPI_F32_ROWS, 4)
QLORA_TC_SMALL(64)
QLORA_TC_SMALL(128)
QLORA_TC_SMALL(192)
QLORA_TC_SMALL(256)

}  // namespace qlora
