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
  int32_t dq;     // 1: q2 codes + group constants; 0: fp32 block scale into absmax
  int32_t dqc;    // scale code (qlora_dq_code_t) when dq
  // cut[j] (j < 15): the real number halfway between m_j (the fp32 midpoint
  // of levels j and j+1) and the next float32 above m_j; a quotient rounds
  // to a float32 above m_j exactly when it exceeds cut[j]. cut[15] is padding.
  double cut[16];
  // Cell table of the encoder: cell c (0..32) holds the quotients x with
  // rint(16 x + 16) == c, widened by twice the guard below; cell_m[c] is the
  // one level midpoint m_j inside the widened cell (4.0 if there is none) and
  // cell_below[c] the number of midpoints below the widened cell (a float).
  // A cell is 1/16 wide and the midpoints are more than 0.08 apart.
  float cell_m[33];
  float cell_below[33];
};
// |fl32(w * r) - fl32(w / s)| < 3.4e-7 for |w| <= s, a normal s below 2^126
// and r within 2 ulp of 1/s; a quotient farther than this guard from the
// candidate midpoint is decided without the exact test.
constexpr float kEncodeGuard = 5e-7f;

struct DequantParams {
  float cb[16];   // the 16 fp32 levels
  int32_t dq;     // 1: s_hat from q2 and the group constants; 0: absmax holds s_b per block
  int32_t dqc;    // scale code (qlora_dq_code_t) when dq: 2 has two constants per group
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
  int32_t dq;             // 1: s_hat from q2 and the group constants; 0: smax holds s_b per block
  int32_t dqc;            // scale code (qlora_dq_code_t) when dq: 2 has two constants per group
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

// NT token groups of 8; SC the block-scale format (kScNone .. kScS8Mid of nf4_dev.cuh)
template <int NT, int SC>
__global__ void k_gemv_nf4(GemvParams p);
template <int MT>
__global__ void k_lora_down_small(LoraDownSmallParams p);

// ------------------------------------------------------------ tensor-core GEMM engine
// Operand sources: A from TMA (K- or MN-major), or the restored NF4 weight
// (K-major for the forward, MN-major for dX); B from TMA.
enum ASrc : int { A_TMA_K = 0, A_TMA_MN = 1, A_DQ_K = 2, A_DQ_MN = 3 };
enum BSrc : int { B_TMA_K = 0, B_TMA_MN = 1 };

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
  int32_t dq;           // 1: s_hat from q2 and the group constants; 0: smax holds s_b per block
  int32_t dqc;          // scale code (qlora_dq_code_t) when dq: 2 has two constants per group
                        // (only with NH = 1: its restore slots have room for both)
  int64_t w_rows;       // N of the weight (rows of W)
  int64_t w_cols;       // K of the weight
  float cb[16];
  // LoRA A operand for the extra k-tiles, copied by the A-producer warps
  const __nv_bfloat16* lora;
  int64_t lora_ld;      // row stride (elements)
  int32_t lora_r;       // valid extent of the LoRA rank
  // output
  void* out;
  int64_t ldo;          // pair kernel: row stride of out [cols x ldo]; small kernel: slabs [split][rows_pad][ldo]
  int32_t rows_pad;     // small kernel: rows per split slab
  int32_t tma_out;      // pair kernel: write the output through TMA stores
  // pair kernel, stream-K schedule (sk = 1; needs tma_out): equal ranges of
  // the (tile, k-tile) space per CTA pair; a tile cut between two pairs goes
  // through one fp32 partial slot per CTA, [128 x 256 NH] floats each, laid
  // out [column / 4][row][4], and four ready flags per CTA (one per epilogue
  // warp), zeroed before the call's first kernel
  int32_t sk;
  float* sk_part;
  uint32_t* sk_flags;
  // pair kernel: features per tile (the MMA's N), a multiple of 16 in
  // [128, 256]; below 256 only for the forward (its restore takes any
  // feature offset; dX slices must stay 64-aligned)
  int32_t feat_n;
};

// TMA-fed tcgen05 GEMM for the small LoRA products: persistent CTAs (at most
// one per SM) walk tile = row tile * splits + split and write fp32 partial
// slabs part[split][rows_pad][ld]; k_reduce_splits finishes them.
struct SmallParams {
  int32_t rows;          // output rows
  int32_t rows_pad;      // tiles * 128
  int32_t ld;            // padded width r64 = BN (slab row stride; mode 0 out_pad row stride)
  int32_t cols;          // valid output columns r
  int32_t tiles;         // 128-row tiles
  int32_t kt_main;       // 64-wide k-tiles of the reduction
  int32_t kt_split;      // k-tiles per split
  int32_t splits;
  float* part;           // [splits][rows_pad][ld] fp32
  float scale;
  int32_t mode;          // 0: bf16 out_pad [rows x ld] and out_c [rows x cols] (if set)
                         // 1: fp32 out_f [rows x cols]; 2: fp32 out_f [cols x rows]
  __nv_bfloat16* out_pad;
  __nv_bfloat16* out_c;
  float* out_f;
};

template <int BN, int AS, int BS, int STAGES>
__global__ void k_tc_small(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                           SmallParams p);

// as many pipeline stages as fit beside the control block, at most eight
constexpr int small_stages(int bn) {
  return (200 * 1024) / (16384 + bn * 128) > 8 ? 8 : (200 * 1024) / (16384 + bn * 128);
}

template <int BN>
constexpr int tc_small_smem_bytes() {
  return small_stages(BN) * (16384 + BN * 128) + 1024 + 256;
}

constexpr int kScalePrefetch = 4;  // k-tiles of scale codes fetched ahead by each restore thread

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

// bytes of scale data per restore thread and k-tile in the pair kernels: the
// q2 word and one group constant (8), or with room for the signed scale
// code's second constant (16; NH = 1 only, NH = 2 has no shared memory left)
constexpr uint32_t pair_scale_slot(int nh) { return nh == 1 ? 16u : 8u; }

constexpr int tc_pair_smem_bytes(int nh) {
  return pair_stages(nh) * (16384 + nh * 16384 + 4096) + 1024 + 256 +
         2 * kScalePrefetch * 128 * static_cast<int>(pair_scale_slot(nh)) + kPairEpiStage;
}

__global__ void k_reduce_splits(SmallParams p);

__global__ void k_selftest_wait(uint64_t limit_ns);

// LoRA merge for export: out = bf16(W_hat + s B A), 128 x 128 tiles.
struct MergeParams {
  const uint8_t* codes;
  const uint8_t* q2;
  const float* smax;
  const __nv_bfloat16* a;   // [r x K]
  const __nv_bfloat16* b;   // [N x r]
  __nv_bfloat16* out;       // [N x K]
  int64_t n, k;
  int32_t r, r64;
  float s;
  int32_t dq;               // 1: s_hat from q2 and the group constants; 0: smax holds s_b per block
  int32_t dqc;              // scale code (qlora_dq_code_t) when dq: 2 has two constants per group
  float cb[16];
  int32_t tiles_n, tiles_k; // tensor-core merge: 128-row x 256-column output tiles
};
__global__ void k_merge_lora(MergeParams p);

// Tensor-core merge (B rows 16-byte aligned, r % 8 == 0): persistent CTAs,
// s B A for a 128 x 256 tile in tensor memory (tcgen05, operands by TMA), the
// restore, add and rounding in the drain, output by TMA stores.
//   tm_b: B [N x r] bf16, boxes {64, 128}; tm_a: A [r x K] bf16, boxes {64, 64};
//   tm_codes: codes [N x K/2] bytes, boxes {128, 128}; tm_out: out [N x K] bf16, boxes {32, 32}
__global__ void k_merge_tc(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_a,
                           const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_out,
                           MergeParams p);
constexpr int kMergeStages = 2;        // operand stages (one 64-rank chunk of B and A each)
constexpr int kMergeCodeStages = 3;    // code tiles in flight
constexpr int kMergeDrainWarps = 16;   // 4 lane quarters x 4 blocks of 64 columns
constexpr size_t merge_tc_smem_bytes() {
  return 1024 + kMergeStages * 49152 + kMergeCodeStages * 16384 + kMergeDrainWarps * 2 * 2048 + 256;
}

// AdamW step over n parameters (fp32 master, grad, m, v; optional bf16 copy).
struct AdamwParams {
  float* master;
  const float* grad;
  float* m;
  float* v;
  __nv_bfloat16* param;     // may be null
  int64_t n;
  float beta1, beta2, eps;
  float decay;              // 1 - lr * weight_decay
  float step_size;          // lr / (1 - beta1^t)
  float inv_sqrt_bc2;       // 1 / sqrt(1 - beta2^t)
  int32_t vec4;             // all pointers 16-byte aligned (param 8-byte)
};
__global__ void k_adamw(AdamwParams a);
inline size_t merge_smem_bytes(int r64) {
  return static_cast<size_t>(128) * (r64 + 8) * 2 + static_cast<size_t>(r64) * 136 * 2 + 128 * 132 * 4;
}

// Device check of the current device (sm_100, attributes set), as every entry
// point runs it: QLORA_OK, QLORA_ERR_UNSUPPORTED_DEVICE or QLORA_ERR_CUDA
// (values of qlora_status_t, returned as int to keep the ABI header out).
int check_current_device_status();

// The calling thread's current CUDA context (nullptr on failure). Entry
// points call it after check_current_device_status, which has made the
// runtime's primary context current.
CUcontext current_context();

// Zero-padded copy of a [rows x r] bf16 matrix into [rows x r64].
__global__ void k_pad_cols(const __nv_bfloat16* __restrict__ src, __nv_bfloat16* __restrict__ dst,
                           int64_t rows, int32_t r, int32_t r64);

}  // namespace qlora
