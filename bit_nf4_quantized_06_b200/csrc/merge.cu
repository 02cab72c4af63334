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
// costs 2 r flops per weight and runs on the tensor cores. One CTA owns a
// 128 x 128 tile of the output:
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

}  // namespace qlora
