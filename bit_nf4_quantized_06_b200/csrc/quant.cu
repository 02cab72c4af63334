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
// or one of the two further scale codes (qlora_dq_code_t in the ABI header:
// the 255-step grid, or the signed code centred on the group's mid-range,
// which also needs the group's minimum scale).
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

// Reciprocal by the hardware approximation (within 2 ulp for the normal
// scales below 2^126 that reach it; the encoder's guard covers that error).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// Shared-memory load at a byte address; volatile keeps it after the barrier
// that publishes the tables.
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}

// 8-byte shared-memory load (cell entry: midpoint, count of midpoints below + 1)
__device__ __forceinline__ uint2 lds_u2(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t abs_bits_max(uint4 v) {
  // bf16 magnitudes compare like unsigned integers once the sign is cleared
  // (a NaN's pattern is above infinity's); both halves at once
  uint32_t m = vmax_u16x2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
  m = vmax_u16x2(m, v.z & 0x7FFF7FFFu);
  m = vmax_u16x2(m, v.w & 0x7FFF7FFFu);
  return max(m & 0xFFFFu, m >> 16);
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
// Encode by cells: with r the hardware reciprocal of s (within 2 ulp of 1 / s
// for a normal s below 2^126), the quotient x' = fl32(w * r) lies within
// 2^-22 + 2^-24 + 2^-25 < 3.4e-7 of fl32(w / s) for |w| <= s. Its cell c = rint(16 x' + 16) (0..32, one fused multiply-add
// around a large constant) selects the one level midpoint m inside the cell
// (a cell is narrower than the gaps between midpoints) and the number of
// midpoints below it, so q = below + [x' > m] -- exactly the count
// #{j : fl32(w / s) > m_j} whenever |x' - m| exceeds the guard. Two weights
// go through each step as a packed fp32 pair (mul / fma .f32x2, each lane
// rounded like the scalar operation): x', the cell's float t, and d^2 - G^2
// whose sign bit says |d| < G for d = x' - m. One 8-byte table entry per
// cell holds m and (midpoints below + 1); the word is the sum of those counts
// at the eight nibble positions minus the sign bits of the eight d's (x' < m
// takes one off), gathered with byte permutes -- d is never zero here, as
// |d| >= G > 0. The table is read at 8 bits(t) + constant. Chunks with a
// quotient within the guard of a midpoint take the exact test above for
// those weights; blocks whose scale is zero, subnormal, at least 2^126 or not
// finite take it (or the value the definition gives) for every weight.
__global__ void __launch_bounds__(256, 3) k_quantize_nf4(const uint4* __restrict__ w,
                                                      int64_t nb, uint32_t* __restrict__ codes,
                                                      uint8_t* __restrict__ q2,
                                                      float* __restrict__ smax, QuantParams qp) {
  __shared__ float s_tab[66];     // [0, 33): the midpoint in each cell; [33, 66): midpoints below it
  __shared__ uint2 s_cell[33];    // per cell: (bits of its midpoint, midpoints below it + 1)
  __shared__ double s_cut[16];
  __shared__ uint32_t s_wmax[8];
  __shared__ uint32_t s_wmin[8];
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
    s_tab[tid] = qp.cell_m[tid];
    s_tab[33 + tid] = qp.cell_below[tid];
    s_cell[tid] = make_uint2(__float_as_uint(qp.cell_m[tid]), static_cast<uint32_t>(qp.cell_below[tid]) + 1u);
  }
  if (tid < 16) s_cut[tid] = qp.cut[tid];

  uint32_t am[8];
  uint32_t gm = 0, gn = 0xFFFFu;   // group max, and min over the group's blocks (not its padding)
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t m = abs_bits_max(v[i]);
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, 4));
    am[i] = m;
    gm = max(gm, m);
    gn = min(gn, ((tid >> 3) + 32 * i < nblk) ? m : 0xFFFFu);
  }
  gm = max(gm, __shfl_xor_sync(0xFFFFFFFFu, gm, 8));
  gm = max(gm, __shfl_xor_sync(0xFFFFFFFFu, gm, 16));
  gn = min(gn, __shfl_xor_sync(0xFFFFFFFFu, gn, 8));
  gn = min(gn, __shfl_xor_sync(0xFFFFFFFFu, gn, 16));
  if ((tid & 31) == 0) {
    s_wmax[tid >> 5] = gm;
    s_wmin[tid >> 5] = gn;
  }
  __syncthreads();
  uint32_t gmax = s_wmax[0], gmin = s_wmin[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) {
    gmax = max(gmax, s_wmax[i]);
    gmin = min(gmin, s_wmin[i]);
  }
  const float s_max = __uint_as_float(gmax << 16);
  // per-block outputs: the eight lanes of a block group each take one of
  // the group's eight blocks, (tid >> 3) + 32 * (tid & 7)
  const int sub = tid & 7;
  uint32_t my_am = am[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) my_am = (sub == i) ? am[i] : my_am;
  const int my_bi = (tid >> 3) + 32 * sub;
  if (!qp.dq) {
    // 4.5-bit format: the block scale itself is stored (exact: a bf16 magnitude)
    if (my_bi < nblk) smax[b0 + my_bi] = __uint_as_float(my_am << 16);
  } else if (qp.dqc == 2) {
    // signed code centred on the group's mid-range: two constants per group
    const float lo = __uint_as_float(gmin << 16);
    const float mid = __fmul_rn(__fadd_rn(lo, s_max), 0.5f);
    const float half = __fmul_rn(__fsub_rn(s_max, lo), 0.5f);
    if (tid == 0) {
      smax[2 * g] = mid;
      smax[2 * g + 1] = half;
    }
    if (my_bi < nblk) {
      int code = 0;
      if (half != 0.0f) {
        const float t = __fsub_rn(__uint_as_float(my_am << 16), mid);
        const float ratio = __fdiv_rn(__fmul_rn(127.0f, t), half);
        code = max(-127, min(127, __float2int_rn(ratio)));
      }
      q2[b0 + my_bi] = static_cast<uint8_t>(static_cast<int8_t>(code));
    }
  } else {
    if (tid == 0) smax[g] = s_max;
    if (my_bi < nblk) {
      uint32_t code = 0;
      if (s_max != 0.0f) {
        // 256 steps (the printed grid; 256 s is exact) or 255 steps
        const float num = qp.dqc == 1 ? __fmul_rn(255.0f, __uint_as_float(my_am << 16))
                                      : 256.0f * __uint_as_float(my_am << 16);
        const float ratio = __fdiv_rn(num, s_max);
        code = static_cast<uint32_t>(min(255, __float2int_rn(ratio)));
      }
      q2[b0 + my_bi] = static_cast<uint8_t>(code);
    }
  }

  constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23: the integer part lands in the low mantissa bits
  // shared address of cell c's midpoint is 4 * bits(t) + tab_base, t = 16 x + 16 + kMagic
  const uint32_t tab_base = smem_u32(s_tab) - __float_as_uint(kMagic) * 4u;
  const uint32_t cell_base = smem_u32(s_cell) - __float_as_uint(kMagic) * 8u;   // cell c at 8 c
  constexpr float kGuard2 = kEncodeGuard * kEncodeGuard;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int bi = (tid >> 3) + 32 * i;
    if (bi < nblk) {
      const uint32_t a = am[i];
      const float sb = __uint_as_float(a << 16);
      // zero, subnormal, >= 2^126 (1/s subnormal), infinite or NaN scale
      const bool edge = (a < 0x0080u) || (a >= 0x7E80u);
      const uint32_t ww[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      uint32_t word = 0;
      bool slow = edge;
      if (!edge) {
        // two weights per step: bf16 pair h holds element 2h (low half, high
        // nibble of byte h) and element 2h + 1 (high half, low nibble)
        const float r = rcp_approx(sb);
        const uint64_t r2 = f2(r, r);
        const uint64_t k16 = f2(16.0f, 16.0f), kc = f2(16.0f + kMagic, 16.0f + kMagic);
        const uint64_t ng2 = f2(-kGuard2, -kGuard2);
        uint32_t dev[4], dod[4];   // bits of x - m for the even and the odd element of each pair
        uint32_t near = 0, bsum = 0;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const uint64_t x2 = f2_mul(f2(__uint_as_float(ww[h] << 16), __uint_as_float(ww[h] & 0xFFFF0000u)), r2);
          uint32_t t0, t1, x0, x1;
          f2_split(f2_fma(x2, k16, kc), t0, t1);        // cells 0..32: |x| <= 1 + 2^-21
          f2_split(x2, x0, x1);
          const uint2 c0 = lds_u2(t0 * 8u + cell_base);
          const uint2 c1 = lds_u2(t1 * 8u + cell_base);
          const float d0 = __fsub_rn(__uint_as_float(x0), __uint_as_float(c0.x));
          const float d1 = __fsub_rn(__uint_as_float(x1), __uint_as_float(c1.x));
          dev[h] = __float_as_uint(d0);
          dod[h] = __float_as_uint(d1);
          // d^2 - G^2 < 0 (sign bit set) exactly when |d| < G
          uint32_t g0, g1;
          f2_split(f2_fma(f2(d0, d1), f2(d0, d1), ng2), g0, g1);
          near |= g0 | g1;
          // each nibble first gets (midpoints below + 1); the code is one less
          // where x is below the cell's midpoint (d < 0)
          bsum += c0.y * (16u << (8 * h)) + c1.y * (1u << (8 * h));
        }
        if (near & 0x80000000u) {
          slow = true;
        } else {
          // sign bits of d: even elements to bits 8h + 4, odd ones to bits 8h
          const uint32_t se = prmt(prmt(dev[0], dev[1], 0x0073u), prmt(dev[2], dev[3], 0x7300u), 0x7610u);
          const uint32_t so = prmt(prmt(dod[0], dod[1], 0x0073u), prmt(dod[2], dod[3], 0x7300u), 0x7610u);
          word = bsum - ((se >> 3) & 0x10101010u) - ((so >> 7) & 0x01010101u);
        }
      }
      if (slow) {
        // rare: the exact test for the weights near a midpoint, or the whole block
        const float r = edge ? 0.0f : rcp_approx(sb);
#pragma unroll 1
        for (int e = 0; e < 8; ++e) {
          const float we = (e & 1) ? __uint_as_float(ww[e >> 1] & 0xFFFF0000u) : __uint_as_float(ww[e >> 1] << 16);
          uint32_t q;
          if (a == 0) {
            q = 7u;                                    // s = 0 stores level 7
          } else if (a >= 0x7F80u) {
            // s = inf: fl32(w / s) = +-0 for finite w (7 midpoints below 0); NaN otherwise,
            // which the definition orders above every midpoint
            q = (a == 0x7F80u && (__float_as_uint(we) & 0x7F800000u) != 0x7F800000u) ? 7u : 15u;
          } else if (edge) {
            q = exact_code(we, sb, s_cut);
          } else {
            const float x = __fmul_rn(we, r);
            const float t = fmaf(x, 16.0f, 16.0f + kMagic);
            const uint32_t addr = __float_as_uint(t) * 4u + tab_base;
            const float d = __fsub_rn(x, lds_f32(addr));
            q = static_cast<uint32_t>(lds_f32(addr + 132u)) + (d > 0.0f ? 1u : 0u);
            if (!(fabsf(d) > kEncodeGuard)) q = exact_code(we, sb, s_cut);
          }
          word |= ((e & 1) ? q : (q << 4)) << (8 * (e >> 1));
        }
      }
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
    float s_hat;
    if (!dp.dq) {
      s_hat = __ldg(smax + b);
    } else if (dp.dqc == 2) {
      s_hat = dq_block_scale(__ldg(q2 + b), __ldg(smax + 2 * (b >> 8)), __ldg(smax + 2 * (b >> 8) + 1), 2);
    } else {
      s_hat = dq_block_scale(__ldg(q2 + b), __ldg(smax + (b >> 8)), 0.0f, dp.dqc);
    }
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
