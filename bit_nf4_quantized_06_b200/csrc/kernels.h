// Internal kernel declarations and parameter blocks (not part of the ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace qlora {

// Device status word: kernels OR in a QLORA_DEV_* bit when a bounded wait
// gives up (defined in quant.cu, read by qlora_device_status()).
extern __device__ unsigned int g_dev_status;

struct QuantParams {
  // cut[j] (j < 15): the real number halfway between m_j (the fp32 midpoint
  // of levels j and j+1) and the next float32 above m_j; a quotient rounds
  // to a float32 above m_j exactly when it exceeds cut[j]. cut[15] is padding.
  double cut[16];
};

struct DequantParams {
  float cb[16];   // the 16 fp32 levels
};

__global__ void k_quantize_nf4(const uint4* __restrict__ w, int64_t nb, uint32_t* __restrict__ codes,
                               uint8_t* __restrict__ q2, float* __restrict__ smax, QuantParams qp);

__global__ void k_dequantize_nf4(const uint32_t* __restrict__ codes, const uint8_t* __restrict__ q2,
                                 const float* __restrict__ smax, int64_t nwords,
                                 uint4* __restrict__ out, DequantParams dp);

// ------------------------------------------------------------ decode GEMV
struct GemvParams {
  const uint8_t* codes;   // [N x K/2]
  const uint8_t* q2;      // [N*K/64]
  const float* smax;      // [groups]
  const __nv_bfloat16* x; // [M x K]
  const __nv_bfloat16* u; // [M x r64] u' = bf16(s x A^T), zero padded
  const __nv_bfloat16* b; // [N x ldb] LoRA up projection
  __nv_bfloat16* y;       // [M x N]
  int64_t n, k;
  int32_t m, r, r64, ldb;
  float cb[16];
};

// u'[m][j] = bf16(s * sum_k x[m][k] a[j][k]) for m < M (M <= 16), j < r64
// (columns r..r64 written as zero); also into u_out [M x r] when non-null.
struct LoraDownSmallParams {
  const __nv_bfloat16* x;  // [M x K]
  const __nv_bfloat16* a;  // [r x K]
  __nv_bfloat16* u_pad;    // [M x r64]
  __nv_bfloat16* u_out;    // [M x r] or null
  int64_t k;
  int32_t m, r, r64;
  float s;
};

template <int NT>
__global__ void k_gemv_nf4(GemvParams p);
__global__ void k_lora_down_small(LoraDownSmallParams p);

// ------------------------------------------------------------ tensor-core GEMM engine
// Operand sources of the generic tcgen05 kernel.
enum ASrc : int { A_TMA_K = 0, A_TMA_MN = 1, A_DQ_K = 2, A_DQ_MN = 3 };
enum BSrc : int { B_TMA_K = 0, B_TMA_MN = 1 };
enum Epi : int { EPI_BF16_T = 0, EPI_F32_ROWS = 1 };

struct TcParams {
  int32_t rows;         // extent of the D rows (TMEM lanes) over the whole grid
  int32_t cols;         // extent of the D columns
  int32_t kt_main;      // main k-tiles (64 each) in the reduction
  int32_t kt_lora;      // extra k-tiles appended after the main ones (LoRA term)
  int32_t kt_split;     // main k-tiles per split
  int32_t tiles_rows;   // 128-row tiles
  int32_t tiles_cols;   // BN-column tiles
  int32_t splits;       // reduction splits (tile index = (row tile * tiles_cols + col tile) * splits + split)
  // restored-weight operand (A_DQ_*)
  const uint8_t* q2;
  const float* smax;
  int64_t kblocks;      // K/64 of the weight: blocks per weight row
  int64_t nblocks;      // N*K/64: length of q2
  int64_t w_rows;       // N of the weight (rows of W)
  int64_t w_cols;       // K of the weight
  float cb[16];
  // LoRA A operand for the extra k-tiles, copied by the A-producer warps
  const __nv_bfloat16* lora;
  int64_t lora_ld;      // row stride (elements)
  int32_t lora_r;       // valid extent of the LoRA rank
  // output
  void* out;
  int64_t ldo;          // EPI_BF16_T: row stride of out [cols x ldo]; EPI_F32_ROWS: [split][rows_pad][ldo]
  int32_t rows_pad;     // EPI_F32_ROWS: rows per split slab
  int32_t tma_out;      // pair kernel: write the output through TMA stores
};

// Persistent kernel: gridDim.x CTAs (at most one per SM) walk the tiles
// blockIdx.x, blockIdx.x + gridDim.x, ...
template <int BN, int AS, int BS, int EP, int STAGES>
__global__ void k_tc_gemm(const __grid_constant__ CUtensorMap tm_a,
                          const __grid_constant__ CUtensorMap tm_b,
                          const __grid_constant__ CUtensorMap tm_b_lora,
                          const __grid_constant__ CUtensorMap tm_codes, TcParams p);

constexpr int kScalePrefetch = 4;  // k-tiles of scale codes fetched ahead by each A-producer thread

template <int AS>
constexpr bool tc_dq() { return AS == A_DQ_K || AS == A_DQ_MN; }

template <int AS>
constexpr int tc_threads() { return tc_dq<AS>() ? 448 : 192; }

template <int BN, int AS, int BS, int STAGES>
constexpr int tc_smem_bytes() {
  return STAGES * (16384 + BN * 128 + (tc_dq<AS>() ? 4096 : 0)) + 1024 + 256 +
         (tc_dq<AS>() ? 2 * kScalePrefetch * 128 * 8 : 0);
}

// CTA-pair (cta_group::2) fused restore + GEMM for the forward (A_DQ_K) and
// dX (A_DQ_MN): clusters of two CTAs walk 256 x (256 NH) tiles; tiles_rows
// counts 256-row tiles and tiles_cols (256 NH)-column tiles. Launched with
// cluster dimension 2.
// NH = token groups of 256 per restored A tile (1 or 2).
constexpr int pair_stages(int nh) { return nh == 1 ? 5 : 4; }
constexpr int kPairEpiStage = 4 * 2048;  // four 32 x 32 bf16 output boxes for TMA stores

// tm_out: bf16 output [tokens x features] with boxes of 32 x 32 and 64-byte
// swizzle; used when p.tma_out != 0 (row stride a multiple of 16 bytes).
template <int AS, int NH>
__global__ void k_tc_pair(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_b_lora,
                          const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_out,
                          TcParams p);

constexpr int tc_pair_smem_bytes(int nh) {
  return pair_stages(nh) * (16384 + nh * 16384 + 4096) + 1024 + 256 + 2 * kScalePrefetch * 128 * 8 +
         kPairEpiStage;
}

// Split reductions (fixed order over splits -> deterministic).
struct ReduceParams {
  const float* part;        // [splits][rows_pad][ld]
  int32_t splits, rows, rows_pad, ld, cols;
  float scale;
  __nv_bfloat16* out_pad;   // mode 0: bf16 [rows x ld]   (all ld columns)
  __nv_bfloat16* out_c;     // mode 0: bf16 [rows x cols] (may be null)
  float* out_f;             // mode 1: fp32 [rows x cols]; mode 2: fp32 [cols x rows] (transposed)
  int32_t mode;
};
__global__ void k_reduce_splits(ReduceParams p);

// Zero-padded copy of a [rows x r] bf16 matrix into [rows x r64].
__global__ void k_pad_cols(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                           int64_t rows, int32_t r, int32_t r64);

}  // namespace qlora
