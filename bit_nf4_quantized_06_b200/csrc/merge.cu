// LoRA merge for export on sm_100a:
//
//   W_merged[n][k] = bf16( W_hat[n][k] + s * sum_j B[n][j] A[j][k] )
//
// ("48GB GPU Fine-Tuning a 65B Model ...", § "LoRA Freezes the Original
// Weights ...": after training B A has the shape of W and is added to it, so
// inference pays nothing extra; § "QLoRA Puts the Two Methods in Different
// Places": with a 4-bit base the adapters go into the restored 16-bit
// weights, not into the codes.)
//
// The pass is bound by HBM: it reads 0.5 byte of codes (plus 1/64 byte of
// scale code) and writes 2 bytes of bf16 per weight, while the rank-r product
// costs 2 r flops per weight and runs on the tensor cores. Two kernels:
// k_merge_tc (below; tcgen05, operands by TMA) when B's rows are 16-byte
// aligned (r % 8 == 0), and k_merge_lora for the other ranks, where one CTA
// owns a 128 x 128 tile of the output:
//   1. B[n0 .. n0+128][0 .. r64) and A[0 .. r64)[k0 .. k0+128) are staged in
//      shared memory (zero past r, N and K);
//   2. eight warps (a 4 x 2 grid of 32 x 64 sub-tiles) form B A with
//      mma.sync m16n8k16 (bf16 in, fp32 accumulate) fed by ldmatrix, and
//      store s * (B A) to a shared fp32 tile;
//   3. every thread then takes 8 consecutive weights of a row at a time
//      (their code word and scale codes were requested at the very start):
//      one 32-bit code word, the block's restored scale, the exact restore
//      w_hat = bf16(fl32(c[q] * s_hat)), one fp32 add, one rounding to bf16,
//      one 16-byte store (fully coalesced along the row).
#include "kernels.h"
#include "nf4_dev.cuh"
#include "ptx.cuh"
#include "tc_common.cuh"

namespace qlora {

namespace {

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3},"
      " {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float bf16_round_f(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

// fl32(w + c) for the bf16 in the low (hi = 0) or high half of `pair`: the
// bf16 operand widens exactly, so this is the fp32 sum rounded to nearest even
__device__ __forceinline__ float add_bf16_f32(uint32_t pair, float c, int hi) {
  float d;
  if (hi)
    asm("{ .reg .b16 l, h; mov.b32 {l, h}, %1; add.rn.f32.bf16 %0, h, %2; }" : "=f"(d) : "r"(pair), "f"(c));
  else
    asm("{ .reg .b16 l, h; mov.b32 {l, h}, %1; add.rn.f32.bf16 %0, l, %2; }" : "=f"(d) : "r"(pair), "f"(c));
  return d;
}

}  // namespace

__global__ void __launch_bounds__(256, 2) k_merge_lora(MergeParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int r64 = p.r64;
  const int ldb = r64 + 8;                        // bf16 elements per staged B row (16-byte pad)
  constexpr int LDA = 128 + 8;                    // bf16 elements per staged A row
  constexpr int LDD = 128 + 4;                    // floats per row of the product tile
  __nv_bfloat16* const sB = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* const sA = sB + 128 * ldb;
  float* const sD = reinterpret_cast<float*>(sA + r64 * LDA);
  __shared__ float s_cb[16];

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * 128;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * 128;
  if (tid < 16) s_cb[tid] = p.cb[tid];

  // the packed weight of this thread's eight 8-weight chunks (step 3) is
  // requested first, so its DRAM latency overlaps the staging and the MMAs
  const int64_t kpr = p.k >> 6;
  uint32_t cw[8];
  uint32_t cq2[8];
  float csm[8], csm2[8];    // group constants (the second only for the signed scale code)
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int c = tid + 256 * it;
    const int row = c >> 4, c8 = c & 15;
    const int64_t n = n0 + row, kc = k0 + c8 * 8;
    cw[it] = 0;
    cq2[it] = 0;
    csm[it] = csm2[it] = 0.0f;
    if (n < p.n && kc < p.k) {
      const int64_t e0 = n * p.k + kc;
      cw[it] = __ldcs(reinterpret_cast<const uint32_t*>(p.codes) + (e0 >> 3));
      const int64_t blk = n * kpr + (kc >> 6);
      if (!p.dq) {
        csm[it] = __ldg(p.smax + blk);     // fp32 block scale, no double quantization
      } else if (p.dqc == 2) {
        cq2[it] = __ldg(p.q2 + blk);
        csm[it] = __ldg(p.smax + 2 * (blk >> 8));
        csm2[it] = __ldg(p.smax + 2 * (blk >> 8) + 1);
      } else {
        cq2[it] = __ldg(p.q2 + blk);
        csm[it] = __ldg(p.smax + (blk >> 8));
      }
    }
  }

  // 1. stage B rows n0.. (r64 columns, zero past r and N) and A columns k0..
  //    (zero past r and K); loads are issued in batches of four before their
  //    stores so that several are in flight per thread
  const int cpr = r64 / 8;                        // 16-byte chunks per staged B row
  if ((p.r & 7) == 0) {
    for (int i0 = tid; i0 < 128 * cpr; i0 += 4 * 256) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * 256;
        const int row = i / cpr, c8 = i - row * cpr;
        v[u] = make_uint4(0, 0, 0, 0);
        if (i < 128 * cpr && n0 + row < p.n && c8 * 8 < p.r)
          v[u] = __ldg(reinterpret_cast<const uint4*>(p.b + (n0 + row) * p.r + c8 * 8));
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * 256;
        const int row = i / cpr, c8 = i - row * cpr;
        if (i < 128 * cpr) *reinterpret_cast<uint4*>(sB + row * ldb + c8 * 8) = v[u];
      }
    }
  } else {
    for (int i0 = tid; i0 < 128 * r64; i0 += 8 * 256) {
      __nv_bfloat16 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * 256;
        const int row = i / r64, j = i - row * r64;
        v[u] = __float2bfloat16_rn(0.0f);
        if (i < 128 * r64 && n0 + row < p.n && j < p.r) v[u] = p.b[(n0 + row) * p.r + j];
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * 256;
        const int row = i / r64, j = i - row * r64;
        if (i < 128 * r64) sB[row * ldb + j] = v[u];
      }
    }
  }
  for (int i0 = tid; i0 < r64 * 16; i0 += 4 * 256) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * 256;
      const int j = i >> 4, c8 = i & 15;
      v[u] = make_uint4(0, 0, 0, 0);
      if (i < r64 * 16 && j < p.r && k0 + c8 * 8 < p.k)
        v[u] = __ldg(reinterpret_cast<const uint4*>(p.a + j * p.k + k0 + c8 * 8));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * 256;
      if (i < r64 * 16) *reinterpret_cast<uint4*>(sA + (i >> 4) * LDA + (i & 15) * 8) = v[u];
    }
  }
  __syncthreads();

  // 2. s * (B A) for this warp's 32 x 64 sub-tile
  {
    const int wm = warp >> 1, wn = warp & 1;
    float acc[2][8][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][j][q] = 0.0f;
    const uint32_t sB_u = smem_u32(sB), sA_u = smem_u32(sA);
    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;
    const int lcol = (lane >> 4) * 8;
    for (int kk = 0; kk < r64; kk += 16) {
      uint32_t af[2][4];
#pragma unroll
      for (int i = 0; i < 2; ++i)
        ldsm_x4(sB_u + 2u * ((32 * wm + 16 * i + lrow) * ldb + kk + lcol), af[i][0], af[i][1], af[i][2], af[i][3]);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sA_u + 2u * ((kk + lrow) * LDA + 64 * wn + 16 * jj + lcol), b0, b1, b2, b3);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          mma16816(acc[i][2 * jj], af[i][0], af[i][1], af[i][2], af[i][3], b0, b1);
          mma16816(acc[i][2 * jj + 1], af[i][0], af[i][1], af[i][2], af[i][3], b2, b3);
        }
      }
    }
    const int g = lane >> 2, qd = lane & 3;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int row = 32 * wm + 16 * i + g;
        const int col = 64 * wn + 8 * j + 2 * qd;
        sD[row * LDD + col] = p.s * acc[i][j][0];
        sD[row * LDD + col + 1] = p.s * acc[i][j][1];
        sD[(row + 8) * LDD + col] = p.s * acc[i][j][2];
        sD[(row + 8) * LDD + col + 1] = p.s * acc[i][j][3];
      }
  }
  __syncthreads();

  // 3. restore, add, round, store: 16 threads per row, 8 weights each
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    const int c = tid + 256 * it;
    const int row = c >> 4, c8 = c & 15;
    const int64_t n = n0 + row, kc = k0 + c8 * 8;
    if (n >= p.n || kc >= p.k) continue;
    const int64_t e0 = n * p.k + kc;                 // first element of the chunk
    const uint32_t w = cw[it];
    const float sh = p.dq ? dq_block_scale(cq2[it], csm[it], csm2[it], p.dqc) : csm[it];
    const float4 dlo = *reinterpret_cast<const float4*>(sD + row * LDD + c8 * 8);
    const float4 dhi = *reinterpret_cast<const float4*>(sD + row * LDD + c8 * 8 + 4);
    const float d[8] = {dlo.x, dlo.y, dlo.z, dlo.w, dhi.x, dhi.y, dhi.z, dhi.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // byte j holds element 2j in its high nibble and 2j+1 in its low nibble
      const uint32_t byte = (w >> (8 * j)) & 0xFFu;
      const float w0 = bf16_round_f(__fmul_rn(s_cb[byte >> 4], sh));
      const float w1 = bf16_round_f(__fmul_rn(s_cb[byte & 15u], sh));
      o[j] = pack_bf16x2(__fadd_rn(w0, d[2 * j]), __fadd_rn(w1, d[2 * j + 1]));
    }
    __stcs(reinterpret_cast<uint4*>(p.out + e0), make_uint4(o[0], o[1], o[2], o[3]));
  }
}

// ---------------------------------------------------------------------------
// Tensor-core merge. Persistent CTAs (one per SM) walk 128-row x 256-column
// output tiles (columns fastest). For each tile
//   D[128 x 256] (fp32, tensor memory) = B[n0 .., 0 .. r64) A[0 .. r64, k0 ..)
// runs on tcgen05 (M 128, N 256, K 16 per instruction), A and B arriving by
// TMA in 64-rank chunks (B K-major, A MN-major, zero past r, N and K), while
// the tile's packed codes arrive by TMA in a 128 x 128-byte swizzled box.
// Sixteen drain warps (lane quarter w % 4, 64-column block (w - 2) / 4: one
// weight block per row) load their 64 accumulator values per row from tensor
// memory and their 32 bytes of codes from shared memory at once, release
// both, and then per 32 columns: the block's 16-entry table (its scale data
// fetched one tile ahead), w_hat = bf16(fl32(c[q] s_hat)) by table lookup,
// fl32(s * acc) for two weights at a time, the add w_hat + that in fp32 (the
// bf16 w_hat widens exactly inside the mixed-precision add), one rounding,
// and a 32 x 32 TMA store. Two accumulators let the drain of one tile
// overlap the products of the next.
//
// Warps: 0 TMA producer (one lane), 1 tensor-memory owner and MMA issuer
// (one lane), 2-17 drain. Every wait is bounded; every TMA load fills only
// this CTA's shared memory.
__global__ void __launch_bounds__(576, 1)
    k_merge_tc(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_a,
               const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_out,
               MergeParams p) {
  using namespace tcd;
  constexpr int STAGES = kMergeStages;
  constexpr int CST = kMergeCodeStages;
  constexpr uint32_t B_BYTES = 16384;          // 128 rows of B x 64 ranks (MMA operand A, K-major)
  constexpr uint32_t A_BYTES = 32768;          // 64 ranks x 256 columns of A (MMA operand B, MN-major)
  constexpr uint32_t STAGE_BYTES = B_BYTES + A_BYTES;
  constexpr uint32_t C_BYTES = 16384;          // 128 rows x 128 bytes of codes
  constexpr uint32_t IDESC = idesc_bf16_f32(128, 256, false, true);
  constexpr uint32_t ACC_COLS = 256;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t codes0 = base + STAGES * STAGE_BYTES;
  const uint32_t epi0 = codes0 + CST * C_BYTES;         // two 2 KB boxes per drain warp
  const uint32_t bar0 = epi0 + kMergeDrainWarps * 2 * 2048;
  uint8_t* const ctl = smem_raw + (bar0 - raw);
  auto bar_full = [&](int s) { return bar0 + 8u * s; };
  auto bar_empty = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto bar_cfull = [&](int c) { return bar0 + 8u * (2 * STAGES + c); };
  auto bar_cempty = [&](int c) { return bar0 + 8u * (2 * STAGES + CST + c); };
  auto bar_accf = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 * CST + b); };
  auto bar_acce = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 * CST + 2 + b); };
  const uint32_t bar_fin = bar0 + 8u * (2 * STAGES + 2 * CST + 4);
  uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(ctl + 8 * (2 * STAGES + 2 * CST + 5));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(ctl + 8 * (2 * STAGES + 2 * CST + 5) + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntiles = p.tiles_n * p.tiles_k;
  const int nchunks = p.r64 / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int c = 0; c < CST; ++c) {
      mbar_init(bar_cfull(c), 1);
      mbar_init(bar_cempty(c), kMergeDrainWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf(b), 1);
      mbar_init(bar_acce(b), kMergeDrainWarps);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_holder), 2 * ACC_COLS);
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
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_codes);
      int it = 0, i = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++i) {
        const int n0 = (tile / p.tiles_k) * 128;
        const int k0 = (tile % p.tiles_k) * 256;
        const int cs = i % CST;
        if (!mbar_wait(bar_cempty(cs), ((i / CST) & 1) ^ 1, abort_flag, QLORA_DEV_TIMEOUT_PRODUCER)) break;
        const uint32_t c_s = codes0 + cs * C_BYTES;
        mbar_arrive_expect_tx(bar_cfull(cs), C_BYTES);
        tma_load_2d(c_s, &tm_codes, bar_cfull(cs), k0 / 2, n0);
        for (int c = 0; c < nchunks; ++c, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(bar_empty(s), ((it / STAGES) & 1) ^ 1, abort_flag, QLORA_DEV_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          const uint32_t b_s = base + s * STAGE_BYTES;
          const uint32_t a_s = b_s + B_BYTES;
          mbar_arrive_expect_tx(bar_full(s), STAGE_BYTES);
          tma_load_2d(b_s, &tm_b, bar_full(s), c * 64, n0);
#pragma unroll
          for (int j = 0; j < 4; ++j) tma_load_2d(a_s + j * 8192, &tm_a, bar_full(s), k0 + 64 * j, c * 64);
        }
      }
      // every load this thread started has landed before the CTA can exit
      for (int j = max(0, it - STAGES); j < it; ++j) drain_wait(bar_full(j % STAGES), (j / STAGES) & 1);
      for (int j = max(0, i - CST); j < i; ++j) drain_wait(bar_cfull(j % CST), (j / CST) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int it = 0, i = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++i) {
        const int b = i & 1;
        if (!mbar_wait(bar_acce(b), ((i >> 1) & 1) ^ 1, abort_flag, QLORA_DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * ACC_COLS;
        for (int c = 0; c < nchunks; ++c, ++it) {
          const int s = it % STAGES;
          if (!mbar_wait(bar_full(s), (it / STAGES) & 1, abort_flag, QLORA_DEV_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b_s = base + s * STAGE_BYTES;
          const uint32_t a_s = b_s + B_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t da = smem_desc_sw128(b_s + kk * 32, 16, 1024);
            const uint64_t db = smem_desc_sw128(a_s + kk * 2048, 8192, 1024);
            tc_mma_ss(d_tmem, da, db, IDESC, (c > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(bar_empty(s));
        }
        if (ok) tc_commit(bar_accf(b));
      }
      tc_commit(bar_fin);
      drain_wait(bar_fin, 0);
    }
  } else {
    // ---------------------------------------------------------------- drain
    const int quarter = warp & 3;          // tensor-memory lanes [32 quarter, +32)
    const int cb = (warp - 2) >> 2;        // columns [64 cb, +64) of the tile: one block per row
    const int row = quarter * 32 + lane;   // this lane's row of the tile
    const int64_t kpr = p.k >> 6;          // blocks per weight row
    const uint32_t box0 = epi0 + (warp - 2) * 4096;
    // raw scale data of this lane's block in a tile (zero past N or K)
    struct ScaleData {
      uint32_t q2;
      float c0, c1;
    };
    auto fetch_scale = [&](int tile) {
      ScaleData d{0u, 0.0f, 0.0f};
      if (tile < ntiles) {
        const int64_t n = (tile / p.tiles_k) * 128 + row;
        const int64_t kc = (tile % p.tiles_k) * 256 + 64 * cb;
        if (n < p.n && kc < p.k) {
          const int64_t blk = n * kpr + (kc >> 6);
          if (!p.dq) {
            d.c0 = __ldg(p.smax + blk);
          } else if (p.dqc == 2) {
            d.q2 = __ldg(p.q2 + blk);
            d.c0 = __ldg(p.smax + 2 * (blk >> 8));
            d.c1 = __ldg(p.smax + 2 * (blk >> 8) + 1);
          } else {
            d.q2 = __ldg(p.q2 + blk);
            d.c0 = __ldg(p.smax + (blk >> 8));
          }
        }
      }
      return d;
    };
    int i = 0, nbox = 0;
    ScaleData nxt = fetch_scale(blockIdx.x);
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++i) {
      const int n0 = (tile / p.tiles_k) * 128;
      const int k0 = (tile % p.tiles_k) * 256;
      const ScaleData cur = nxt;
      nxt = fetch_scale(tile + gridDim.x);   // in flight while this tile drains
      const float sh = p.dq ? dq_block_scale(cur.q2, cur.c0, cur.c1, p.dqc) : cur.c0;
      const int cs = i % CST;
      const int b = i & 1;
      bool ok = mbar_wait(bar_cfull(cs), (i / CST) & 1, abort_flag, QLORA_DEV_TIMEOUT_EPI);
      if (ok) ok = mbar_wait(bar_accf(b), (i >> 1) & 1, abort_flag, QLORA_DEV_TIMEOUT_EPI);
      if (!warp_all(ok)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + b * ACC_COLS + (static_cast<uint32_t>(quarter * 32) << 16) + 64 * cb;
      const uint32_t crow = codes0 + cs * C_BYTES + row * 128;
      const Nf4Table tb = make_table(p.cb, sh);
      const uint64_t s2 = f2(p.s, p.s);
      uint32_t acc0[32], acc1[32];
      tmem_ld_32x32b_x32(taddr, acc0);
      tmem_ld_32x32b_x32(taddr + 32, acc1);
      const uint4 cw0 = lds128(crow + ((((cb << 1) + 0) ^ (row & 7)) << 4));
      const uint4 cw1 = lds128(crow + ((((cb << 1) + 1) ^ (row & 7)) << 4));
      tc_wait_ld();
      // every accumulator column and code word of this warp is in registers
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar_acce(b));
        mbar_arrive(bar_cempty(cs));
      }
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        const uint32_t* acc = ch ? acc1 : acc0;
        const uint4 cw = ch ? cw1 : cw0;
        const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
        uint32_t o[16];
#pragma unroll
        for (int wd = 0; wd < 4; ++wd) {
          uint32_t wh[4];
          lookup8(tb, words[wd], wh);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // fl32(s * acc) for both weights of the pair at once, then
            // w_hat + that with the bf16 w_hat widened inside the add
            uint32_t d0, d1;
            f2_split(f2_mul(s2, f2(__uint_as_float(acc[8 * wd + 2 * j]), __uint_as_float(acc[8 * wd + 2 * j + 1]))),
                     d0, d1);
            o[4 * wd + j] = pack_bf16x2(add_bf16_f32(wh[j], __uint_as_float(d0), 0),
                                        add_bf16_f32(wh[j], __uint_as_float(d1), 1));
          }
        }
        const int x = k0 + 64 * cb + 32 * ch;
        if (x < p.k) {
          // stage the 32 x 32 chunk (64-byte swizzle) in the box the store
          // before last used, once that store has read it, and store it
          const uint32_t box = box0 + (nbox & 1) * 2048;
          if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
          __syncwarp();
          const uint32_t rw = box + lane * 64;
          const uint32_t sw = (lane >> 1) & 3;
#pragma unroll
          for (int v = 0; v < 4; ++v)
            sts128(rw + ((v ^ sw) << 4), o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tm_out, box, x, n0 + quarter * 32);
            bulk_commit();
          }
          ++nbox;
        }
      }
    }
    if (lane == 0) bulk_wait_all();   // stores complete before the CTA's shared memory goes away
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * ACC_COLS);
  }
}

}  // namespace qlora
