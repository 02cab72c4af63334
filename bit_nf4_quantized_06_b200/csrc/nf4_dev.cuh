// Device-side NF4 restore helpers shared by the tensor-core GEMMs and the
// decode GEMV.
//
// Restore rule ("48GB GPU Fine-Tuning a 65B Model ...", § "Quantization Keeps
// the Patterns and Reduces Bits per Number": multiply the level by the block
// scale, compute in bf16; «QLoRA는 어떻게 65B 모델을 GPU 한 장에 올렸나»,
// § "메모리 회계": c(q) * q2/256 * s_max):
//
//     s_hat = fl32(q2 * s_max) * 2^-8
//     w_hat = bf16_rne(fl32(c[q] * s_hat))
//
// Within one 64-weight block s_hat is constant, so the 16 possible restored
// values are computed once per block (16 fp32 multiplies, 8 packed bf16
// conversions) and every weight is then a table lookup. The table is kept as
// two byte planes (low bytes, high bytes of the 16 bf16 values) in 8
// registers, so a lookup is a byte permute: prmt picks 4 bytes out of an
// 8-byte register pair by 3-bit indices, one pair for levels 0..7 and one for
// 8..15, merged by bit 3 of each index. The result is bit-identical to
// computing each weight on its own.
#pragma once

#include "ptx.cuh"

namespace qlora {

struct Nf4Table {
  uint32_t lo[4];  // low bytes of entries 4i..4i+3
  uint32_t hi[4];  // high bytes of entries 4i..4i+3
};

__device__ __forceinline__ float restored_scale(uint32_t q2, float smax) {
  const float prod = __fmul_rn(static_cast<float>(q2), smax);
  return __fmul_rn(prod, 0.00390625f);  // 2^-8, exact except for subnormal results
}

// Block scale of a scale code (qlora_dq_code_t; the formulas of the ABI
// header): c0 = s_max (or mid), c1 = half (signed code only).
__device__ __forceinline__ float dq_block_scale(uint32_t q2, float c0, float c1, int code) {
  if (code == 1) return __fdiv_rn(__fmul_rn(static_cast<float>(q2), c0), 255.0f);
  if (code == 2) {
    const float q = static_cast<float>(static_cast<int>(static_cast<int8_t>(static_cast<uint8_t>(q2))));
    return __fadd_rn(c0, __fdiv_rn(__fmul_rn(q, c1), 127.0f));
  }
  return restored_scale(q2, c0);
}

// Block-scale format as a compile-time constant, for kernels instantiated
// per format: no double quantization (fp32 block scales), or one of the
// three scale codes (qlora_dq_code_t + 1).
constexpr int kScNone = 0, kScU8x256 = 1, kScU8x255 = 2, kScS8Mid = 3;

__host__ __device__ constexpr int scale_format(int dq, int dqc) { return dq ? dqc + 1 : kScNone; }

// Restored block scale for format SC: c0 is the fp32 block scale (kScNone)
// or the group constant (s_max, or mid for kScS8Mid with c1 = half).
template <int SC>
__device__ __forceinline__ float block_scale_sc(uint32_t q2, float c0, float c1) {
  if constexpr (SC == kScNone) {
    return c0;
  } else {
    return dq_block_scale(q2, c0, c1, SC - 1);
  }
}

// cb: the 16 fp32 levels (kernel-parameter constants).
__device__ __forceinline__ Nf4Table make_table(const float (&cb)[16], float s_hat) {
  uint32_t p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    p[i] = pack_bf16x2(__fmul_rn(cb[2 * i], s_hat), __fmul_rn(cb[2 * i + 1], s_hat));
  Nf4Table t;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    t.lo[i] = prmt(p[2 * i], p[2 * i + 1], 0x6420);
    t.hi[i] = prmt(p[2 * i], p[2 * i + 1], 0x7531);
  }
  return t;
}

// One 32-bit word of packed codes (bytes little-endian, byte i holds element
// 2i in its high nibble and 2i+1 in its low nibble) -> 8 restored bf16 values
// as 4 packed pairs out[j] = (element 2j in the low half, 2j+1 in the high).
__device__ __forceinline__ void lookup8(const Nf4Table& t, uint32_t w, uint32_t (&out)[4]) {
  const uint32_t sel = w & 0x77777777u;         // 3-bit index per nibble
  const uint32_t sel_hi = sel >> 16;
  const uint32_t w4 = w << 4;
  // 0xFF in byte p where nibble p of w has bit 3 set (levels 8..15);
  // prmt's sign-replicate mode copies bit 7 of the chosen source byte.
  const uint32_t m0 = prmt(w4, w, 0xD9C8);
  const uint32_t m1 = prmt(w4, w, 0xFBEA);
  // nibble order in w: p = 0..7 -> elements 1,0,3,2,5,4,7,6
  uint32_t lo0 = lop3_sel(prmt(t.lo[0], t.lo[1], sel), prmt(t.lo[2], t.lo[3], sel), m0);
  uint32_t hi0 = lop3_sel(prmt(t.hi[0], t.hi[1], sel), prmt(t.hi[2], t.hi[3], sel), m0);
  uint32_t lo1 = lop3_sel(prmt(t.lo[0], t.lo[1], sel_hi), prmt(t.lo[2], t.lo[3], sel_hi), m1);
  uint32_t hi1 = lop3_sel(prmt(t.hi[0], t.hi[1], sel_hi), prmt(t.hi[2], t.hi[3], sel_hi), m1);
  out[0] = prmt(lo0, hi0, 0x4051);  // (e0, e1)
  out[1] = prmt(lo0, hi0, 0x6273);  // (e2, e3)
  out[2] = prmt(lo1, hi1, 0x4051);  // (e4, e5)
  out[3] = prmt(lo1, hi1, 0x6273);  // (e6, e7)
}

}  // namespace qlora
