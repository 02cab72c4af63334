// Generic tcgen05 GEMM engine for sm_100a, one 128 x BN output tile per CTA.
//
//   D[128 x BN] (fp32, in tensor memory)  +=  A[128 x 64] * B[BN x 64]^T  per k-tile
//
// Warp roles (192 threads):
//   warp 0    one lane issues TMA loads (B tiles, A tiles when A comes from
//             memory, packed NF4 code tiles when A is restored on chip)
//   warp 1    allocates tensor memory; one lane issues tcgen05.mma and commits
//   warps 2-5 A producers when A is a restored NF4 weight: per stage they turn
//             the staged 4-bit codes into bf16 directly in the 128-byte
//             swizzled shared-memory layout the tensor core reads (K-major
//             for the forward, MN-major for dX); for the appended LoRA
//             k-tiles they copy the adapter rows instead. Afterwards the same
//             four warps drain the accumulator (tcgen05.ld) and write it out.
//
// The forward pass ("48GB GPU Fine-Tuning a 65B Model ...", § "QLoRA Puts the
// Two Methods in Different Places": each block of W is restored to bf16,
// multiplied with the input, and the LoRA branch is added) runs with
// D = y^T tile: rows are output features, columns are tokens, A = restored W,
// B = x, and s * u' * B_lora^T appended as extra k-tiles of the same
// accumulator. dX uses D = dX^T tile with A = restored W seen MN-major
// (the 4-bit blocks run along d_in, the reduction runs along d_out) and
// B = dY, plus s * v' * A_lora as extra k-tiles. The small LoRA products
// (x A^T, dY B, dA, dB) reuse the same kernel with both operands from TMA.
//
// Every pipeline wait is bounded (see ptx.cuh); no TMA load uses cluster
// multicast.
#include "kernels.h"
#include "nf4_dev.cuh"
#include "ptx.cuh"

namespace qlora {

namespace {

__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xFFFFFFFFu, v); }

__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity) {
  // wait that ignores the abort flag: used only to let in-flight async work
  // land before the CTA releases its shared and tensor memory
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > QLORA_WAIT_LIMIT_NS) return false;
  }
  return true;
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

template <int BN>
constexpr uint32_t tmem_cols() {
  return BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
}

}  // namespace

template <int BN, int AS, int BS, int EP, int STAGES>
__global__ void __launch_bounds__(192, 1)
    k_tc_gemm(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
              const __grid_constant__ CUtensorMap tm_b_lora,
              const __grid_constant__ CUtensorMap tm_codes, TcParams p) {
  constexpr bool DQ = (AS == A_DQ_K || AS == A_DQ_MN);
  constexpr bool A_MN = (AS == A_TMA_MN || AS == A_DQ_MN);
  constexpr bool B_MN = (BS == B_TMA_MN);
  constexpr uint32_t A_BYTES = 16384;
  constexpr uint32_t B_BYTES = BN * 128;
  constexpr uint32_t C_BYTES = DQ ? 4096 : 0;
  constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + C_BYTES;
  constexpr uint32_t IDESC = idesc_bf16_f32(128, BN, A_MN, B_MN);
  constexpr uint32_t TMEM_COLS = tmem_cols<BN>();
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* const base_ptr = smem_raw + (base - raw);
  uint8_t* const ctl = base_ptr + STAGES * STAGE_BYTES;
  const uint32_t bar0 = base + STAGES * STAGE_BYTES;
  // barriers: full[S] (TMA bytes), codes[S] (TMA bytes), afull[S] (A producers),
  //           empty[S] (MMA commit), acc (MMA commit)
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_codes = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto bar_afull = [&](int s) { return bar0 + 8u * (2 * STAGES + s); };
  auto bar_empty = [&](int s) { return bar0 + 8u * (3 * STAGES + s); };
  const uint32_t bar_acc = bar0 + 8u * (4 * STAGES);
  uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(ctl + 8 * (4 * STAGES + 1));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(ctl + 8 * (4 * STAGES + 1) + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int row0 = blockIdx.x * 128;
  const int col0 = blockIdx.y * BN;
  const int kt_begin = blockIdx.z * p.kt_split;
  const int kt_end = min(p.kt_main, kt_begin + p.kt_split);
  const int nmain = max(0, kt_end - kt_begin);
  const int ntiles = nmain + p.kt_lora;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_codes(s), 1);
      mbar_init(bar_afull(s), 4);
      mbar_init(bar_empty(s), 1);
    }
    mbar_init(bar_acc, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), TMEM_COLS);
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
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % STAGES;
        const uint32_t ph = (t / STAGES) & 1;
        if (!mbar_wait(bar_empty(s), ph ^ 1, abort_flag, QLORA_DEV_TIMEOUT_PRODUCER)) break;
        const uint32_t a_s = base + s * STAGE_BYTES;
        const uint32_t b_s = a_s + A_BYTES;
        const uint32_t c_s = b_s + B_BYTES;
        if (t < nmain) {
          const int kt = kt_begin + t;
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
          const int lt = t - nmain;
          mbar_arrive_expect_tx(bar_full(s), B_BYTES);
          tma_load_2d(b_s, &tm_b_lora, bar_full(s), lt * 64, col0);
        }
        issued = t + 1;
      }
      // let every load this thread started land before the CTA can exit
      for (int t = max(0, issued - STAGES); t < issued; ++t) {
        drain_wait(bar_full(t % STAGES), (t / STAGES) & 1);
        if (DQ && t < nmain) drain_wait(bar_codes(t % STAGES), (t / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % STAGES;
        const uint32_t ph = (t / STAGES) & 1;
        if (!mbar_wait(bar_full(s), ph, abort_flag, QLORA_DEV_TIMEOUT_MMA)) break;
        if (DQ && !mbar_wait(bar_afull(s), ph, abort_flag, QLORA_DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t a_s = base + s * STAGE_BYTES;
        const uint32_t b_s = a_s + A_BYTES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t da = A_MN ? smem_desc_sw128(a_s + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(a_s + kk * 32, 16, 1024);
          const uint64_t db = B_MN ? smem_desc_sw128(b_s + kk * 2048, 8192, 1024)
                                   : smem_desc_sw128(b_s + kk * 32, 16, 1024);
          tc_mma_ss(tmem_base, da, db, IDESC, (t > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar_empty(s));
      }
      tc_commit(bar_acc);
      drain_wait(bar_acc, 0);
    }
  } else {
    const int tid = threadIdx.x - 64;  // 0..127
    // ---------------------------------------------------------------- A producers
    if (DQ) {
      for (int t = 0; t < ntiles; ++t) {
        const int s = t % STAGES;
        const uint32_t ph = (t / STAGES) & 1;
        const uint32_t a_s = base + s * STAGE_BYTES;
        const uint32_t c_s = a_s + A_BYTES + B_BYTES;
        bool ok = mbar_wait(bar_empty(s), ph ^ 1, abort_flag, QLORA_DEV_TIMEOUT_APROD);
        if (!warp_all(ok)) break;
        if (AS == A_DQ_K) {
          // row r of the tile = weight row n; 64 weights = one block
          const int r = tid;
          const int64_t n = row0 + r;
          const uint32_t dst = a_s + r * 128;
          const uint32_t sw = r & 7;
          if (t < nmain) {
            const int kt = kt_begin + t;
            float sh = 0.0f;
            if (n < p.w_rows) {
              const int64_t bi = n * p.kblocks + kt;
              sh = restored_scale(__ldg(p.q2 + bi), __ldg(p.smax + (bi >> 8)));
            }
            const Nf4Table tb = make_table(p.cb, sh);
            ok = mbar_wait(bar_codes(s), ph, abort_flag, QLORA_DEV_TIMEOUT_APROD);
            if (!warp_all(ok)) break;
            const uint4 c0 = lds128(c_s + r * 32);
            const uint4 c1 = lds128(c_s + r * 32 + 16);
            const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
            for (int w = 0; w < 8; ++w) {
              uint32_t o[4];
              lookup8(tb, words[w], o);
              sts128(dst + ((w ^ sw) << 4), o[0], o[1], o[2], o[3]);
            }
          } else {
            const int lt = t - nmain;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint4 v = make_uint4(0, 0, 0, 0);
              const int j = lt * 64 + 8 * c;
              if (n < p.w_rows && j < p.lora_r)
                v = __ldg(reinterpret_cast<const uint4*>(p.lora + n * p.lora_ld + j));
              sts128(dst + ((c ^ sw) << 4), v.x, v.y, v.z, v.w);
            }
          }
        } else {
          // MN-major: tile row nr = reduction index (weight row n), half hh
          // = which 64 of the 128 weight columns [row0, row0 + 128)
          const int nr = tid >> 1;
          const int hh = tid & 1;
          const int64_t kcol = row0 + 64 * hh;
          const bool kvalid = kcol < p.w_cols;
          const uint32_t dst = a_s + hh * 8192 + nr * 128;
          const uint32_t sw = nr & 7;
          if (t < nmain) {
            const int kt = kt_begin + t;
            const int64_t n = static_cast<int64_t>(kt) * 64 + nr;
            float sh = 0.0f;
            if (kvalid && n < p.w_rows) {
              const int64_t bi = n * p.kblocks + (kcol >> 6);
              sh = restored_scale(__ldg(p.q2 + bi), __ldg(p.smax + (bi >> 8)));
            }
            const Nf4Table tb = make_table(p.cb, sh);
            ok = mbar_wait(bar_codes(s), ph, abort_flag, QLORA_DEV_TIMEOUT_APROD);
            if (!warp_all(ok)) break;
            const uint4 c0 = lds128(c_s + nr * 64 + hh * 32);
            const uint4 c1 = lds128(c_s + nr * 64 + hh * 32 + 16);
            const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
            for (int w = 0; w < 8; ++w) {
              uint32_t o[4];
              lookup8(tb, words[w], o);
              sts128(dst + ((w ^ sw) << 4), o[0], o[1], o[2], o[3]);
            }
          } else {
            const int lt = t - nmain;
            const int j = lt * 64 + nr;
            const bool valid = kvalid && j < p.lora_r;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint4 v = make_uint4(0, 0, 0, 0);
              if (valid) v = __ldg(reinterpret_cast<const uint4*>(p.lora + j * p.lora_ld + kcol + 8 * c));
              sts128(dst + ((c ^ sw) << 4), v.x, v.y, v.z, v.w);
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_afull(s));
      }
    }
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes [32 q, 32 q + 32) belong to warp % 4
    bool ok = mbar_wait(bar_acc, 0, abort_flag, QLORA_DEV_TIMEOUT_EPI);
    ok = warp_all(ok);
    tc_fence_after();
    if (ok) {
      const int prow = row0 + quarter * 32 + lane;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
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
              if (q < p.cols) out[static_cast<int64_t>(q) * p.ldo + prow] = __float2bfloat16_rn(__uint_as_float(r[i]));
            }
          }
        } else {
          float* out = reinterpret_cast<float*>(p.out) +
                       (static_cast<int64_t>(blockIdx.z) * p.rows_pad + prow) * p.ldo + col0 + ch * 32;
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(out)[i] =
                make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                            __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
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
