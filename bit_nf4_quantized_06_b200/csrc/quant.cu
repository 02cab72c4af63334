// NF4 blockwise quantizer with double quantization, and the standalone
// restore, for sm_100a.
//
// Quantizer ("48GB GPU Fine-Tuning a 65B Model ...", § "Quantization Keeps
// the Patterns and Reduces Bits per Number"; «QLoRA는 어떻게 65B 모델을 GPU
// 한 장에 올렸나», § "메모리 회계"):
//   s_b   = max |w| over 64 consecutive weights of the row-major matrix
//   q     = #{ j : fl32(w / s_b) > m_j }   (m_j = fp32 midpoints of the levels;
//            an exact tie goes to the lower level; s_b == 0 stores level 7),
//            evaluated without a division (see k_quantize_nf4)
//   byte  = (q[2i] << 4) | q[2i+1]
//   s_max = max s_b over 256 consecutive blocks (the last group may be short)
//   q2    = min(255, rint_even(fl32(256 * s_b / s_max)))   (0 if s_max == 0)
//
// One CTA of 256 threads owns one double-quantization group (256 blocks,
// 16384 weights, 32 KB of bf16): every thread loads 8 x 16 B with fully
// coalesced warp accesses (lane l reads bytes [16 l, 16 l + 16) of each
// 512-byte warp slice), the 8 lanes that share a block reduce its absmax
// with xor shuffles, the group maximum goes through shared memory, and each
// 8-weight chunk is encoded and written back as one 32-bit word, again
// coalesced. W is read exactly once; codes, scale codes and s_max are
// written exactly once.
#include "ptx.cuh"
#include "nf4_dev.cuh"
#include "kernels.h"

namespace qlora {

__device__ unsigned int g_dev_status = 0;

namespace {

__device__ __forceinline__ uint32_t abs_bits_max(uint4 v) {
  // bf16 magnitudes compare like unsigned integers once the sign is cleared
  uint32_t m = 0;
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m = max(m, w[i] & 0x7FFFu);
    m = max(m, (w[i] >> 16) & 0x7FFFu);
  }
  return m;
}

// Exact code of one weight by the division-free test: for a bf16 weight w
// and a block scale s > 0,
//   fl32(w / s) > m_j   <=>   w / s > m'_j   <=>   w > m'_j * s   <=>   w > RD_bf16(m'_j * s)
// where m'_j (cut[j]) is the midpoint between m_j and the next float32 above
// it. Round-to-nearest sends w / s above m_j exactly when w / s exceeds that
// midpoint; equality would need m'_j * s (a 25-bit odd significand times an
// 8-bit one) to have at most 8 significant bits, which it cannot; m'_j * s is
// exact in float64; and because w lies on the bf16 grid, comparing with the
// product rounded down to that grid gives the same answer.
__device__ __noinline__ uint32_t exact_code(float w, float s, const double* cut) {
  uint32_t q = 0;
  for (int j = 0; j < 15; ++j) {
    const float t = __bfloat162float(__float2bfloat16_rd(__double2float_rd(cut[j] * static_cast<double>(s))));
    q += (w > t) ? 1u : 0u;
  }
  return q;
}

}  // namespace

// One CTA of 256 threads per double-quantization group (see the file comment).
//
// Encode by cells: with r = fl32(1 / s), the quotient x' = fl32(w * r) lies
// within 3.0001 * 2^-24 of fl32(w / s) for |w| <= s. Its cell
// c = rint(16 x' + 16) (0..32, one fused multiply-add around a large
// constant) selects a table entry holding the number of level midpoints
// below the cell and the one midpoint m inside it (a cell is narrower than
// the gaps between midpoints), so q = below + [x' > m] -- exactly the count
// #{j : fl32(w / s) > m_j} whenever |x' - m| exceeds the guard. The two
// 33-word tables sit in shared memory, one word per bank, so the lookups
// never conflict. The rare weights within the guard of a midpoint, and
// blocks whose scale is subnormal (1/s may overflow), take the exact test
// above.
__global__ void __launch_bounds__(256, 3) k_quantize_nf4(const uint4* __restrict__ w,
                                                      int64_t nb, uint32_t* __restrict__ codes,
                                                      uint8_t* __restrict__ q2,
                                                      float* __restrict__ smax, QuantParams qp) {
  __shared__ float s_cm[33];
  __shared__ uint32_t s_ci[33];
  __shared__ double s_cut[16];
  __shared__ uint32_t s_wmax[8];
  const int tid = threadIdx.x;
  const int64_t g = blockIdx.x;
  const int64_t b0 = g * 256;
  const int nblk = static_cast<int>(nb - b0 < 256 ? nb - b0 : 256);
  const int64_t chunk0 = b0 * 8;  // 8 chunks of 8 weights per block

  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int bi = (tid >> 3) + 32 * i;
    v[i] = (bi < nblk) ? __ldcs(w + chunk0 + tid + 256 * i) : make_uint4(0, 0, 0, 0);
  }
  if (tid < 33) {
    s_cm[tid] = qp.cell_m[tid];
    s_ci[tid] = qp.cell_info[tid];
  }
  if (tid < 16) s_cut[tid] = qp.cut[tid];

  uint32_t am[8];
  uint32_t gm = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t m = abs_bits_max(v[i]);
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
    am[i] = m;
    gm = max(gm, m);
  }
  gm = max(gm, __shfl_xor_sync(0xFFFFFFFFu, gm, 8));
  gm = max(gm, __shfl_xor_sync(0xFFFFFFFFu, gm, 16));
  if ((tid & 31) == 0) s_wmax[tid >> 5] = gm;
  __syncthreads();
  uint32_t gmax = s_wmax[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) gmax = max(gmax, s_wmax[i]);
  const float s_max = __uint_as_float(gmax << 16);
  if (!qp.dq) {
    // 4.5-bit format: the block scale itself is stored (exact: a bf16 magnitude)
    if ((tid & 7) == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int bi = (tid >> 3) + 32 * i;
        if (bi < nblk) smax[b0 + bi] = __uint_as_float(am[i] << 16);
      }
    }
  } else if (tid == 0) {
    smax[g] = s_max;
  }

  if (qp.dq && (tid & 7) == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int bi = (tid >> 3) + 32 * i;
      if (bi < nblk) {
        uint32_t code = 0;
        if (s_max != 0.0f) {
          const float sb = __uint_as_float(am[i] << 16);
          const float ratio = __fdiv_rn(256.0f * sb, s_max);
          code = static_cast<uint32_t>(min(255, __float2int_rn(ratio)));
        }
        q2[b0 + bi] = static_cast<uint8_t>(code);
      }
    }
  }

  constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23: the integer part lands in the low mantissa bits
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int bi = (tid >> 3) + 32 * i;
    if (bi < nblk) {
      const uint32_t a = am[i];
      const float sb = __uint_as_float(a << 16);
      const bool zero = (a == 0);
      const bool tiny = (a < 0x0080u);     // zero or subnormal scale
      const float r = tiny ? 0.0f : __frcp_rn(sb);
      const uint32_t ww[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      uint32_t qv[8];
      bool any_amb = false;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        // element e of the chunk: bf16 pair e/2 holds element 2k in its low half
        const float we = (e & 1) ? __uint_as_float(ww[e >> 1] & 0xFFFF0000u) : __uint_as_float(ww[e >> 1] << 16);
        const float x = __fmul_rn(we, r);
        const float t = fmaf(x, 16.0f, 16.0f + kMagic);
        const uint32_t c = min(__float_as_uint(t) - __float_as_uint(kMagic), 32u);
        const float d = __fsub_rn(x, s_cm[c]);
        qv[e] = (s_ci[c] & 0xFFu) + (d > 0.0f ? 1u : 0u);
        any_amb |= !(fabsf(d) > kEncodeGuard);
      }
      if (tiny || any_amb) {
        // rare: redo the weights near a midpoint (or the whole block) exactly
#pragma unroll 1
        for (int e = 0; e < 8; ++e) {
          const float we = (e & 1) ? __uint_as_float(ww[e >> 1] & 0xFFFF0000u) : __uint_as_float(ww[e >> 1] << 16);
          if (zero) {
            qv[e] = 7u;
          } else if (tiny) {
            qv[e] = exact_code(we, sb, s_cut);
          } else {
            const float x = __fmul_rn(we, r);
            const float t = fmaf(x, 16.0f, 16.0f + kMagic);
            const uint32_t c = min(__float_as_uint(t) - __float_as_uint(kMagic), 32u);
            if (!(fabsf(__fsub_rn(x, s_cm[c])) > kEncodeGuard)) qv[e] = exact_code(we, sb, s_cut);
          }
        }
      }
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) word |= ((qv[2 * j] << 4) | qv[2 * j + 1]) << (8 * j);
      codes[chunk0 + tid + 256 * i] = word;
    }
  }
}

// Restore: one thread per 8 weights (one 32-bit code word -> one 16-byte
// store). Grid-stride over all words.
__global__ void __launch_bounds__(256) k_dequantize_nf4(const uint32_t* __restrict__ codes,
                                                        const uint8_t* __restrict__ q2,
                                                        const float* __restrict__ smax,
                                                        int64_t nwords, uint4* __restrict__ out,
                                                        DequantParams dp) {
  __shared__ float s_cb[16];
  if (threadIdx.x < 16) s_cb[threadIdx.x] = dp.cb[threadIdx.x];
  __syncthreads();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < nwords;
       i += stride) {
    const int64_t b = i >> 3;
    const float s_hat = dp.dq ? restored_scale(__ldg(q2 + b), __ldg(smax + (b >> 8))) : __ldg(smax + b);
    const uint32_t w = __ldcs(codes + i);
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t byte = (w >> (8 * j)) & 0xFFu;
      const float v0 = __fmul_rn(s_cb[byte >> 4], s_hat);
      const float v1 = __fmul_rn(s_cb[byte & 15u], s_hat);
      o[j] = pack_bf16x2(v0, v1);
    }
    __stcs(out + i, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

// Failure-detection self test: one thread waits on a shared-memory barrier
// that expects one arrival nobody makes. The wait is bounded by `limit_ns`
// of global time; when it runs out the kernel records the self-test bit and
// returns, with nothing in flight (no copies, no tensor memory).
__global__ void __launch_bounds__(32) k_selftest_wait(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_mbar_init();
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(b, 0)) {
      if (globaltimer_ns() - t0 > limit_ns) {
        atomicOr(&g_dev_status, QLORA_DEV_TIMEOUT_SELFTEST);
        break;
      }
    }
  }
}

}  // namespace qlora
