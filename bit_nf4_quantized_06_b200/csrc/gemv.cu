// Decode-sized forward (M <= 16 tokens) for sm_100a.
//
//   y[m][n] = sum_k x[m][k] w_hat[n][k] + sum_j u'[m][j] B[n][j],
//   u'      = bf16(s * x A^T)          (k_lora_down_small, launched first)
//
// At M <= 16 the forward is a stream over the packed weight: 0.5 byte per
// weight plus 1/64 byte of scale code, so it is bound by HBM bandwidth as
// long as restoring a weight costs only a few instructions. Each warp owns
// 16 weight rows; each lane restores whole 64-weight blocks (one table of 16
// bf16 values per block, then one byte-permute lookup per weight, see
// nf4_dev.cuh) straight into the A fragments of mma.sync m16n8k16, with the
// tokens as the 8-wide N side. Because a dot product may visit k in any
// order, the lane's 8 consecutive weights are placed into fragment slots in
// the order they come out of the lookup and x is fetched in the same order,
// so no shuffle is needed. The eight warps of a CTA split K; their partial
// fragments are summed in a fixed order in shared memory. The LoRA term is
// appended as r/16 further MMA steps spread over the warps; each warp fetches
// the next chunk's codes and scale codes while it restores the current one,
// and both kernels use programmatic dependent launch: x A^T may launch while
// the kernel before it drains, waits for it, and then lets the GEMV start;
// the GEMV streams the whole weight while x A^T runs beside it and waits for
// x A^T only before the LoRA-up step that reads u'. The GEMV is instantiated
// per block-scale format (no double quantization, or one of the three scale
// codes), so the restore of one format carries no code for the others.
#include "kernels.h"
#include "nf4_dev.cuh"

namespace qlora {

namespace {

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3},"
      " {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ld_bf16_pair(const __nv_bfloat16* row, int j, int r) {
  // (row[j], row[j+1]) with zeros past r; 2-byte loads so any r works
  const uint16_t* p = reinterpret_cast<const uint16_t*>(row);
  const uint32_t lo = (j < r) ? p[j] : 0u;
  const uint32_t hi = (j + 1 < r) ? p[j + 1] : 0u;
  return lo | (hi << 16);
}

}  // namespace

template <int NT, int SC>
__global__ void __launch_bounds__(256, 2) k_gemv_nf4(GemvParams p) {
  constexpr int WARPS = 8;
  __shared__ float s_red[WARPS][32][NT * 4];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int qd = lane & 3;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * 16;
  const int64_t r0 = n0 + g;
  const int64_t r1 = n0 + g + 8;
  const bool v0 = r0 < p.n;
  const bool v1 = r1 < p.n;
  const int64_t kpr = p.k >> 6;
  const int64_t nchunks = (kpr + 3) >> 2;
  const int64_t row_bytes = p.k >> 1;

  float acc[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[t][i] = 0.0f;

  // LoRA-up fragments of this warp's rank steps (j0 = 16 * (warp + 8 i)):
  // inputs of the call, so they are fetched before anything else
  const __nv_bfloat16* brow0 = p.b + (v0 ? r0 : 0) * static_cast<int64_t>(p.ldb);
  const __nv_bfloat16* brow1 = p.b + (v1 ? r1 : 0) * static_cast<int64_t>(p.ldb);
  const int rv0 = v0 ? p.r : 0;
  const int rv1 = v1 ? p.r : 0;
  uint32_t la[2][4];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int ja = 16 * (warp + WARPS * i) + 2 * qd;
    la[i][0] = ld_bf16_pair(brow0, ja, rv0);
    la[i][1] = ld_bf16_pair(brow1, ja, rv1);
    la[i][2] = ld_bf16_pair(brow0, ja + 8, rv0);
    la[i][3] = ld_bf16_pair(brow1, ja + 8, rv1);
  }

  // one chunk = 4 blocks (256 weights) of both rows; lane (g, qd) owns block qd
  struct Chunk {
    uint4 a_lo, a_hi, b_lo, b_hi;
    uint32_t q2a, q2b;
    float sma, smb, sma2, smb2;   // group constants (the second only for the signed scale code)
  };
  // the group constants of block bi (dq) or its fp32 scale (no dq)
  auto scale_data = [&](int64_t bi, uint32_t& q2, float& c0, float& c1) {
    if constexpr (SC == kScNone) {
      c0 = __ldg(p.smax + bi);          // fp32 block scale, no double quantization
    } else if constexpr (SC == kScS8Mid) {
      q2 = __ldg(p.q2 + bi);
      c0 = __ldg(p.smax + 2 * (bi >> 8));
      c1 = __ldg(p.smax + 2 * (bi >> 8) + 1);
    } else {
      q2 = __ldg(p.q2 + bi);
      c0 = __ldg(p.smax + (bi >> 8));
    }
  };
  auto fetch = [&](int64_t c, Chunk& ch) {
    const int64_t kb = c * 4 + qd;
    const bool kv = c < nchunks && kb < kpr;
    ch.a_lo = ch.a_hi = ch.b_lo = ch.b_hi = make_uint4(0, 0, 0, 0);
    ch.q2a = ch.q2b = 0;
    ch.sma = ch.smb = ch.sma2 = ch.smb2 = 0.0f;
    if (kv && v0) {
      const uint8_t* src = p.codes + r0 * row_bytes + kb * 32;
      ch.a_lo = ldg_stream(src);
      ch.a_hi = ldg_stream(src + 16);
      scale_data(r0 * kpr + kb, ch.q2a, ch.sma, ch.sma2);
    }
    if (kv && v1) {
      const uint8_t* src = p.codes + r1 * row_bytes + kb * 32;
      ch.b_lo = ldg_stream(src);
      ch.b_hi = ldg_stream(src + 16);
      scale_data(r1 * kpr + kb, ch.q2b, ch.smb, ch.smb2);
    }
  };

  // x A^T, the kernel launched just before this one, starts only after all
  // earlier work is complete and writes nothing but u'; so everything except
  // u' may be read at once, and u' only after waiting for that kernel.
  Chunk cur, nxt;
  fetch(warp, cur);
  fetch(warp + WARPS, nxt);
  grid_dependency_trigger();
  for (int64_t c = warp; c < nchunks; c += WARPS) {
    const int64_t kb = c * 4 + qd;
    const bool kv = kb < kpr;
    const Nf4Table t0 = make_table(p.cb, block_scale_sc<SC>(cur.q2a, cur.sma, cur.sma2));
    const Nf4Table t1 = make_table(p.cb, block_scale_sc<SC>(cur.q2b, cur.smb, cur.smb2));
    const uint32_t wa[8] = {cur.a_lo.x, cur.a_lo.y, cur.a_lo.z, cur.a_lo.w,
                            cur.a_hi.x, cur.a_hi.y, cur.a_hi.z, cur.a_hi.w};
    const uint32_t wb[8] = {cur.b_lo.x, cur.b_lo.y, cur.b_lo.z, cur.b_lo.w,
                            cur.b_hi.x, cur.b_hi.y, cur.b_hi.z, cur.b_hi.w};
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t ra[4], rb[4];
      lookup8(t0, wa[w], ra);
      lookup8(t1, wb[w], rb);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const int tok = t * 8 + g;
        uint4 xv = make_uint4(0, 0, 0, 0);
        if (kv && tok < p.m)
          xv = __ldg(reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(tok) * p.k + kb * 64 + 8 * w));
        // slots: logical k (2qd, 2qd+1) <- weights 4h+0, 4h+1; (2qd+8, 2qd+9) <- 4h+2, 4h+3
        mma_bf16_16816(acc[t], ra[0], rb[0], ra[1], rb[1], xv.x, xv.y);
        mma_bf16_16816(acc[t], ra[2], rb[2], ra[3], rb[3], xv.z, xv.w);
      }
    }
    cur = nxt;
    fetch(c + 2 * WARPS, nxt);      // loads of the chunk after next fly while the next one is restored
  }

  // LoRA term: sum_j u'[tok][j] B[n][j], 16 ranks per MMA step, steps spread
  // over the warps. u' comes from the kernel in front: wait for it here.
  grid_dependency_wait();
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int j0 = 16 * (warp + WARPS * i);
    if (j0 < p.r64) {
      const int ja = j0 + 2 * qd;
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const int tok = t * 8 + g;
        uint32_t b0 = 0, b1 = 0;
        if (tok < p.m) {
          const uint32_t* urow = reinterpret_cast<const uint32_t*>(p.u + static_cast<int64_t>(tok) * p.r64);
          b0 = urow[ja >> 1];
          b1 = urow[(ja + 8) >> 1];
        }
        mma_bf16_16816(acc[t], la[i][0], la[i][1], la[i][2], la[i][3], b0, b1);
      }
    }
  }

#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) s_red[warp][lane][t * 4 + i] = acc[t][i];
  __syncthreads();
  if (warp != 0) return;
#pragma unroll
  for (int t = 0; t < NT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v = 0.0f;
#pragma unroll
      for (int wv = 0; wv < WARPS; ++wv) v += s_red[wv][lane][t * 4 + i];
      acc[t][i] = v;
    }

#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int tok = t * 8 + 2 * qd;
    if (v0) {
      if (tok < p.m) p.y[static_cast<int64_t>(tok) * p.n + r0] = __float2bfloat16_rn(acc[t][0]);
      if (tok + 1 < p.m) p.y[static_cast<int64_t>(tok + 1) * p.n + r0] = __float2bfloat16_rn(acc[t][1]);
    }
    if (v1) {
      if (tok < p.m) p.y[static_cast<int64_t>(tok) * p.n + r1] = __float2bfloat16_rn(acc[t][2]);
      if (tok + 1 < p.m) p.y[static_cast<int64_t>(tok + 1) * p.n + r1] = __float2bfloat16_rn(acc[t][3]);
    }
  }
}

template __global__ void k_gemv_nf4<1, kScNone>(GemvParams);
template __global__ void k_gemv_nf4<1, kScU8x256>(GemvParams);
template __global__ void k_gemv_nf4<1, kScU8x255>(GemvParams);
template __global__ void k_gemv_nf4<1, kScS8Mid>(GemvParams);
template __global__ void k_gemv_nf4<2, kScNone>(GemvParams);
template __global__ void k_gemv_nf4<2, kScU8x256>(GemvParams);
template __global__ void k_gemv_nf4<2, kScU8x255>(GemvParams);
template __global__ void k_gemv_nf4<2, kScS8Mid>(GemvParams);

// u'[m][j] = bf16(s * sum_k x[m][k] A[j][k]) for M <= 16 (the decode LoRA
// down projection). Rank j is owned by four warps (one per quarter of K)
// whose lanes take 8-element chunks; a shuffle tree and a fixed-order sum of
// the four quarters finish it (deterministic). MT = 1: 16 CTAs of 16 warps
// (4 ranks per CTA per pass); MT > 1: one CTA of 4 warps per rank. Kept
// small in SMs so that the GEMV behind it fits on the GPU beside it and
// streams its weights meanwhile. It waits for everything in front of it
// before reading anything and only then lets the GEMV start, so the GEMV may
// read x without waiting.
template <int MT>
__global__ void __launch_bounds__(MT == 1 ? 512 : 128, MT == 1 ? 2 : 1) k_lora_down_small(LoraDownSmallParams p) {
  __shared__ float s_q[16][MT];     // per warp: partial sums of its quarter
  grid_dependency_wait();
  grid_dependency_trigger();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ranks_per_pass = (MT == 1) ? 4 * gridDim.x : gridDim.x;
  const int rank_in_cta = warp >> 2;
  const int quarter = warp & 3;
  const int64_t nch = p.k >> 3;
  const int64_t q0 = nch * quarter / 4, q1 = nch * (quarter + 1) / 4;
  for (int jb = 0; jb < p.r64; jb += ranks_per_pass) {
    const int j = jb + ((MT == 1) ? blockIdx.x * 4 + rank_in_cta : blockIdx.x);
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
    if (j < p.r) {
      const uint4* arow = reinterpret_cast<const uint4*>(p.a + static_cast<int64_t>(j) * p.k);
      constexpr int kUnroll = MT == 1 ? 4 : (MT == 8 ? 2 : 1);
#pragma unroll kUnroll
      for (int64_t c = q0 + lane; c < q1; c += 32) {
        const uint4 av = __ldg(arow + c);
        const uint32_t aw[4] = {av.x, av.y, av.z, av.w};
        float af[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          af[2 * i] = __uint_as_float(aw[i] << 16);
          af[2 * i + 1] = __uint_as_float(aw[i] & 0xFFFF0000u);
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (m < p.m) {
            const uint4 xv = __ldg(reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(m) * p.k) + c);
            const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              acc[m] = fmaf(af[2 * i], __uint_as_float(xw[i] << 16), acc[m]);
              acc[m] = fmaf(af[2 * i + 1], __uint_as_float(xw[i] & 0xFFFF0000u), acc[m]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xFFFFFFFFu, acc[m], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int m = 0; m < MT; ++m) s_q[warp][m] = acc[m];
    }
    __syncthreads();
    // the first warp of each rank's four sums their quarters in order; lane m writes token m
    if (quarter == 0 && lane < MT && lane < p.m && j < p.r64) {
      const int m = lane;
      const float v = ((s_q[warp][m] + s_q[warp + 1][m]) + s_q[warp + 2][m]) + s_q[warp + 3][m];
      const __nv_bfloat16 b = __float2bfloat16_rn(j < p.r ? v * p.s : 0.0f);
      p.u_pad[static_cast<int64_t>(m) * p.r64 + j] = b;
      if (p.u_out != nullptr && j < p.r) p.u_out[static_cast<int64_t>(m) * p.r + j] = b;
    }
    __syncthreads();
  }
}

template __global__ void k_lora_down_small<1>(LoraDownSmallParams);
template __global__ void k_lora_down_small<8>(LoraDownSmallParams);
template __global__ void k_lora_down_small<16>(LoraDownSmallParams);

}  // namespace qlora
