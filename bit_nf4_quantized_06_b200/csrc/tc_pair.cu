// Fused NF4-restore + tcgen05 GEMM on CTA pairs (cta_group::2), sm_100a.
//
// A cluster of two CTAs computes a (256 NH) tokens x FN features tile of the
// output (y for the forward, dX for the backward), accumulating in fp32 in
// tensor memory with tokens on the tensor-memory lanes:
//
//   D_h[256 tokens x FN features] += T_h[256 x 64] * W[FN x 64]^T   per k-tile, h < NH
//
// FN = 256, or for the data-parallel forward a narrower multiple of 16 that
// fills the last wave better (11008 features: 46 tiles of 240 instead of 43
// of 256, 4.97 waves of 74 pairs instead of 4.65); each CTA then restores
// FN / 2 features (its 128 restore rows past them are ignored by the MMA).
//
// T_h is a 256-token slice of the input (x or dY), loaded by TMA, 128 tokens
// per CTA. W is the 256-feature slice of the restored weight: CTA r restores
// features [FN/2 r, FN/2 r + 128) from the packed codes into the 128-byte
// swizzled layout the tensor core reads (K-major for the forward, MN-major
// for dX, whose reduction runs along d_out while the 4-bit blocks run along
// d_in). The even CTA issues the pair MMAs, which read both CTAs' shared
// memory; each restored W tile serves 256 NH tokens. The LoRA term is appended
// as extra k-tiles of the same accumulators: T = u' (or v') from TMA and
// W = B_lora rows (or A_lora rows) copied by the restore warps.
// ("48GB GPU Fine-Tuning a 65B Model ...", § "QLoRA Puts the Two Methods in
// Different Places": each block of W is restored to bf16 before it meets the
// input, and gradients reach x through the restored W; W gets none.)
//
// With tokens on the lanes, each epilogue warp owns 32 output rows; every
// 32 x 32 chunk goes out as one TMA tensor store from a small swizzled box.
// NH = 2 uses the whole tensor memory for one tile, so the next tile's MMAs
// wait until the drain has read the accumulator (not until the stores are
// done); NH = 1 keeps two accumulators and overlaps the drain entirely.
//
// Warp roles in each CTA (448 threads):
//   warp 0      TMA: this CTA's token slices (completion counted on the even
//               CTA's barrier) and this CTA's code tile (local barrier)
//   warp 1      tensor-memory allocation for the pair; in the even CTA one
//               lane issues the pair MMAs and commits to both CTAs' barriers
//   warps 2-9   restore: two groups of four warps take alternate k-tiles
//   warps 10-13 epilogue: drain this CTA's 128 token rows
//
// Schedules. Data-parallel: pair q takes tiles q, q + npairs, ... . When the
// tile count is not a multiple of the pair count the last wave leaves pairs
// idle; the stream-K schedule (p.sk) keeps all but the last full wave
// data-parallel (the pairs then run in step and share their input tiles in
// L2) and cuts the flattened (tile, k-tile) space of the remaining tiles --
// between one and two waves' worth -- into one equal contiguous range per
// pair. A range that ends inside a tile computes that tile's first k-tiles
// (HEAD) and stores the fp32 partial sums in its slot; the next pair, whose
// range starts inside that tile, computes the remaining k-tiles (TAIL), waits
// for the slot's flags, adds the partial sums in its epilogue and writes the
// tile. A pair processes its HEAD first and its TAIL only once it has done at
// least as many k-tiles as the HEAD it depends on (plus a margin), so the wait
// is normally already over; the writer always has the lower pair index.
//
// Every wait is bounded; every TMA load fills only the issuing CTA's shared
// memory; the MMA's completion reaches the odd CTA through a commit to its
// barrier's cluster address.
#include "kernels.h"
#include "nf4_dev.cuh"
#include "pair_sched.h"
#include "ptx.cuh"
#include "tc_common.cuh"

namespace qlora {

using namespace tcd;
using namespace psched;


template <int AS, int NH>
__global__ void __launch_bounds__(448, 1)
    k_tc_pair(const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_t_lora,
              const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_out,
              TcParams p) {
  constexpr int STAGES = pair_stages(NH);
  constexpr bool W_MN = (AS == A_DQ_MN);
  constexpr uint32_t W_BYTES = 16384;        // 128 features x 64 k, bf16 (restored here)
  constexpr uint32_t T_HALF = 16384;         // 128 tokens x 64 k, bf16 (this CTA's share of one MMA)
  constexpr uint32_t T_BYTES = NH * T_HALF;
  constexpr uint32_t C_BYTES = 4096;         // packed codes for the 128 features
  constexpr uint32_t STAGE_BYTES = W_BYTES + T_BYTES + C_BYTES;
  const int FN = p.feat_n;                   // features per tile (multiple of 16, 128..256)
  const uint32_t idesc = idesc_bf16_f32(256, FN, false, W_MN);
  constexpr uint32_t TILE_COLS = 256 * NH;   // accumulator columns per tile
  constexpr int NBUF = (NH == 1) ? 2 : 1;    // accumulator buffers (double-buffered when they fit)
  constexpr uint32_t TMEM_ALLOC = 512;
  constexpr int PD = kScalePrefetch;
  static_assert(NBUF * TILE_COLS <= TMEM_ALLOC, "tensor memory");
  static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t epi_stage = base + STAGES * STAGE_BYTES;  // 2 KB output box per epilogue warp (1024-aligned)
  uint8_t* const ctl = smem_raw + (base - raw) + STAGES * STAGE_BYTES + kPairEpiStage;
  const uint32_t bar0 = epi_stage + kPairEpiStage;
  auto bar_full = [&](int s) { return bar0 + 8u * s; };                 // even CTA: token slices of both
  auto bar_codes = [&](int s) { return bar0 + 8u * (STAGES + s); };     // local code tile
  auto bar_wfull = [&](int s) { return bar0 + 8u * (2 * STAGES + s); }; // even CTA: 8 restore warps
  auto bar_empty = [&](int s) { return bar0 + 8u * (3 * STAGES + s); }; // local, from the MMA
  auto bar_accf = [&](int b) { return bar0 + 8u * (4 * STAGES + b); };  // local, from the MMA
  auto bar_acce = [&](int b) { return bar0 + 8u * (4 * STAGES + 2 + b); };  // even CTA: 8 epilogue warps
  const uint32_t bar_fin = bar0 + 8u * (4 * STAGES + 4);
  uint32_t* const tmem_holder = reinterpret_cast<uint32_t*>(ctl + 8 * (4 * STAGES + 5));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(ctl + 8 * (4 * STAGES + 5) + 4);
  const uint32_t ring = bar0 + 256;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = (rank == 0);
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;
  const int ntile_total = p.tiles_rows * p.tiles_cols;  // 256-feature x (256 NH)-token tiles
  const PairWork work = make_work(pair, npairs, ntile_total, p.kt_main + p.kt_lora, p.sk != 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_codes(s), 1);
      mbar_init(bar_wfull(s), 8);
      mbar_init(bar_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_accf(b), 1);
      mbar_init(bar_acce(b), 8);
    }
    mbar_init(bar_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), TMEM_ALLOC);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();   // barriers initialised and tensor memory allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // launched as a programmatic dependent: the set-up above overlapped the
  // kernel in front; its results are visible from here on
  grid_dependency_wait();
  grid_dependency_trigger();

  // tile -> first feature of this CTA's restored slice, first token of the tile
  auto tile_feat = [&](int tile) { return (tile / p.tiles_cols) * FN + (FN >> 1) * static_cast<int>(rank); };
  auto tile_tok = [&](int tile) { return (tile % p.tiles_cols) * static_cast<int>(TILE_COLS); };

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_t);
      tma_prefetch_desc(&tm_codes);
      if (p.kt_lora > 0) tma_prefetch_desc(&tm_t_lora);
      int it = 0;
      bool ok = true;
      for (int i = 0; ok && i < work.nseg; ++i) {
        const Seg sg = seg_at(work, i);
        const int f0 = tile_feat(sg.tile);
        const int tok = tile_tok(sg.tile) + 128 * static_cast<int>(rank);
        for (int t = sg.k0; t < sg.k1; ++t, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(bar_empty(s), ph ^ 1, abort_flag, QLORA_DEV_TIMEOUT_PRODUCER)) {
            ok = false;
            break;
          }
          const uint32_t w_s = base + s * STAGE_BYTES;
          const uint32_t t_s = w_s + W_BYTES;
          const uint32_t c_s = t_s + T_BYTES;
          const uint32_t full_even = mapa_shared(bar_full(s), 0);
          if (leader) mbar_arrive_expect_tx(bar_full(s), 2 * T_BYTES);
          if (t < p.kt_main) {
#pragma unroll
            for (int h = 0; h < NH; ++h) tma_load_2d_pair(t_s + h * T_HALF, &tm_t, full_even, t * 64, tok + 256 * h);
            mbar_arrive_expect_tx(bar_codes(s), C_BYTES);
            if (AS == A_DQ_K)
              tma_load_2d(c_s, &tm_codes, bar_codes(s), t * 32, f0);
            else
              tma_load_2d(c_s, &tm_codes, bar_codes(s), f0 / 2, t * 64);
          } else {
#pragma unroll
            for (int h = 0; h < NH; ++h)
              tma_load_2d_pair(t_s + h * T_HALF, &tm_t_lora, full_even, (t - p.kt_main) * 64, tok + 256 * h);
            mbar_arrive(bar_codes(s));  // keeps the code barrier's phase in step
          }
        }
      }
      // the loads this thread started have landed once the MMA released their stage
      for (int j = max(0, it - STAGES); j < it; ++j) {
        drain_wait(bar_empty(j % STAGES), (j / STAGES) & 1);
        drain_wait(bar_codes(j % STAGES), (j / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (even CTA)
    if (leader && lane == 0) {
      int it = 0;
      bool ok = true;
      for (int i = 0; ok && i < work.nseg; ++i) {
        const Seg sg = seg_at(work, i);
        const int b = i % NBUF;
        const uint32_t aph = (i / NBUF) & 1;
        if (!mbar_wait(bar_acce(b), aph ^ 1, abort_flag, QLORA_DEV_TIMEOUT_MMA)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * TILE_COLS;
        for (int t = sg.k0; t < sg.k1; ++t, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (!mbar_wait(bar_full(s), ph, abort_flag, QLORA_DEV_TIMEOUT_MMA) ||
              !mbar_wait(bar_wfull(s), ph, abort_flag, QLORA_DEV_TIMEOUT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t w_s = base + s * STAGE_BYTES;
          const uint32_t t_s = w_s + W_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t dw = W_MN ? smem_desc_sw128(w_s + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(w_s + kk * 32, 16, 1024);
#pragma unroll
            for (int h = 0; h < NH; ++h) {
              const uint64_t dt = smem_desc_sw128(t_s + h * T_HALF + kk * 32, 16, 1024);
              tc_mma_pair(d_tmem + h * 256, dt, dw, idesc, (t > sg.k0 || kk > 0) ? 1u : 0u);
            }
          }
          tc_commit_pair(bar_empty(s));
          tc_commit_pair(mapa_shared(bar_empty(s), 1));
        }
        if (ok) {
          tc_commit_pair(bar_accf(b));
          tc_commit_pair(mapa_shared(bar_accf(b), 1));
        }
      }
      tc_commit_pair(bar_fin);
      drain_wait(bar_fin, 0);
    }
  } else if (warp < 10) {
    // ---------------------------------------------------------------- restore
    const int grp = (warp - 2) >> 2;                 // 0: warps 2-5, 1: warps 6-9
    const int tid = threadIdx.x - 64 - 128 * grp;    // 0..127
    const int items = work.items;
    // scale slot per thread and k-tile: the q2 word and the group constant(s)
    // (the signed scale code's two constants need the 16-byte slot of NH = 1)
    constexpr uint32_t SLOT = pair_scale_slot(NH);
    const uint32_t slot0 = ring + grp * (PD * 128 * SLOT) + tid * SLOT;

    // cursor over this group's items j = grp, grp + 2, ... of the pair's
    // work list: k-tile t (< k1) of segment i, whose restored slice starts at
    // feature f0
    struct Cursor {
      int j, i, t, k1, f0;
    };
    auto settle = [&](Cursor& c) {
      while (c.i < work.nseg && c.t >= c.k1) {
        const int over = c.t - c.k1;
        if (++c.i >= work.nseg) break;
        const Seg sg = seg_at(work, c.i);
        c.t = sg.k0 + over;
        c.k1 = sg.k1;
        c.f0 = tile_feat(sg.tile);
      }
    };
    auto advance = [&](Cursor& c) {
      c.j += 2;
      c.t += 2;
      settle(c);
    };
    // this thread's weight block for k-tile t (-1 = padding)
    auto block_of = [&](int f0, int t) -> int64_t {
      if (AS == A_DQ_K) {
        const int64_t n = f0 + tid;
        return (n < p.w_rows) ? n * p.kblocks + t : -1;
      } else {
        const int64_t n = static_cast<int64_t>(t) * 64 + (tid >> 1);
        const int64_t kcol = f0 + 64 * (tid & 1);
        return (n < p.w_rows && kcol < p.w_cols) ? n * p.kblocks + (kcol >> 6) : -1;
      }
    };
    auto issue = [&](const Cursor& c, int k) {
      if (c.j < items && c.t < p.kt_main) {
        const int64_t bi = block_of(c.f0, c.t);
        const uint32_t slot = slot0 + k * (128 * SLOT);
        if (bi >= 0 && p.dq) {
          const int64_t w4 = bi & ~int64_t(3);
          const int64_t left = p.nblocks - w4;
          cp_async4(slot, p.q2 + w4, static_cast<uint32_t>(left < 4 ? left : 4));
          if (SLOT == 16 && p.dqc == 2) {
            cp_async4(slot + 4, p.smax + 2 * (bi >> 8), 4);
            cp_async4(slot + 8, p.smax + 2 * (bi >> 8) + 1, 4);
          } else {
            cp_async4(slot + 4, p.smax + (bi >> 8), 4);
          }
        } else if (bi >= 0) {
          cp_async4(slot, p.smax, 0);
          cp_async4(slot + 4, p.smax + bi, 4);     // fp32 block scale, no double quantization
        } else {
          cp_async4(slot, p.smax, 0);
          cp_async4(slot + 4, p.smax, 0);
        }
      }
      cp_async_commit();
    };

    Cursor cur{};
    {
      const Seg sg0 = seg_at(work, 0);
      cur = Cursor{grp, 0, sg0.k0 + grp, sg0.k1, tile_feat(sg0.tile)};
      settle(cur);
    }
    Cursor pre = cur;
#pragma unroll 1
    for (int k = 0; k < PD - 1; ++k) {
      issue(pre, k);
      advance(pre);
    }
    int slot_use = 0, slot_issue = PD - 1;
    const uint32_t wfull_even0 = mapa_shared(bar_wfull(0), 0);

#pragma unroll 1
    for (; cur.j < items; advance(cur)) {
      issue(pre, slot_issue);
      advance(pre);
      slot_issue = (slot_issue + 1 == PD) ? 0 : slot_issue + 1;
      const int j = cur.j;
      const int s = j % STAGES;
      const uint32_t ph = (j / STAGES) & 1;
      const int t = cur.t;
      const int f0 = cur.f0;
      const uint32_t w_s = base + s * STAGE_BYTES;
      const uint32_t c_s = w_s + W_BYTES + T_BYTES;
      bool ok = mbar_wait(bar_empty(s), ph ^ 1, abort_flag, QLORA_DEV_TIMEOUT_APROD);
      if (!warp_all(ok)) break;
      if (t < p.kt_main) {
        cp_async_wait<PD - 1>();
        const int64_t bi = block_of(f0, t);
        const uint32_t slot = slot0 + slot_use * (128 * SLOT);
        float sh = 0.0f;
        if (bi >= 0) {
          if (p.dq) {
            const uint32_t qw = lds32(slot);
            const uint32_t q2 = (qw >> (8 * static_cast<uint32_t>(bi & 3))) & 0xFFu;
            const float c1 = (SLOT == 16 && p.dqc == 2) ? __uint_as_float(lds32(slot + 8)) : 0.0f;
            sh = dq_block_scale(q2, __uint_as_float(lds32(slot + 4)), c1, p.dqc);
          } else {
            sh = __uint_as_float(lds32(slot + 4));
          }
        }
        const Nf4Table tb = make_table(p.cb, sh);
        ok = mbar_wait(bar_codes(s), ph, abort_flag, QLORA_DEV_TIMEOUT_APROD);
        if (!warp_all(ok)) break;
        uint32_t src, dst, sw;
        if (AS == A_DQ_K) {
          src = c_s + tid * 32;
          dst = w_s + tid * 128;
          sw = tid & 7;
        } else {
          const int nr = tid >> 1;
          src = c_s + nr * 64 + (tid & 1) * 32;
          dst = w_s + (tid & 1) * 8192 + nr * 128;
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
          const int64_t n = f0 + tid;
          const uint32_t dst = w_s + tid * 128;
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
          const int64_t kcol = f0 + 64 * (tid & 1);
          const bool valid = kcol < p.w_cols && jr < p.lora_r;
          const uint32_t dst = w_s + (tid & 1) * 8192 + nr * 128;
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
      if (lane == 0) {
        if (leader)
          mbar_arrive(bar_wfull(s));
        else
          mbar_arrive_cluster(wfull_even0 + 8u * s);
      }
    }
    cp_async_wait<0>();
  } else {
    // ---------------------------------------------------------------- epilogue
    // Each warp owns 32 token rows (its tensor-memory lane quarter). With
    // TMA stores (row stride a multiple of 16 bytes) every 32 x 32 chunk is
    // converted to bf16, staged in this warp's 2 KB box in the 64-byte
    // swizzled layout (conflict-free for the row-per-lane writes) and written
    // by one bulk tensor store; the accumulator is released as soon as its
    // last chunk has been read. Otherwise each lane stores its row directly.
    const int quarter = warp & 3;  // TMEM lanes [32 q, 32 q + 32) belong to warp % 4
    const uint32_t acce_even0 = mapa_shared(bar_acce(0), 0);
    const bool vec_ok = (p.ldo % 8) == 0;
    const uint32_t box = epi_stage + (warp - 10) * 2048;
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
    // stream-K partial slots hold float4 (column / 4, row) at [column / 4][row]
    const int prow = quarter * 32 + lane;
    constexpr int NCH = TILE_COLS / 32;
    for (int si = 0; si < work.nseg; ++si) {
      const Seg sg = seg_at(work, si);
      const int tile = sg.tile;
      const int b = si % NBUF;
      const uint32_t aph = (si / NBUF) & 1;
      bool ok = mbar_wait(bar_accf(b), aph, abort_flag, QLORA_DEV_TIMEOUT_EPI);
      if (!warp_all(ok)) break;
      tc_fence_after();
      const int f0 = (tile / p.tiles_cols) * FN;    // first feature of the pair's tile
      const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t tbase = tmem_base + b * TILE_COLS + lane_base;
      auto release_acc = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (leader)
            mbar_arrive(bar_acce(b));
          else
            mbar_arrive_cluster(acce_even0 + 8u * b);
        }
      };
      if (sg.kind == SEG_HEAD) {
        // partial sums of the tile's first k-tiles -> this CTA's slot, then
        // this warp's ready flag (release after every lane's stores)
        float4* slot = reinterpret_cast<float4*>(p.sk_part + static_cast<size_t>(blockIdx.x) * (128 * TILE_COLS)) + prow;
        auto store8 = [&](int ch, const uint32_t (&r)[32]) {
#pragma unroll
          for (int v = 0; v < 8; ++v)
            slot[(ch * 8 + v) * 128] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                                   __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
        };
        uint32_t ra[32], rb[32];
        tmem_ld_32x32b_x32(tbase, ra);
        tc_wait_ld();
#pragma unroll 1
        for (int ch = 0; ch < NCH; ch += 2) {
          tmem_ld_32x32b_x32(tbase + (ch + 1) * 32, rb);
          store8(ch, ra);
          tc_wait_ld();
          if (ch + 2 < NCH) tmem_ld_32x32b_x32(tbase + (ch + 2) * 32, ra);
          store8(ch + 1, rb);
          if (ch + 2 < NCH) tc_wait_ld();
        }
        release_acc();
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          st_release_gpu(p.sk_flags + blockIdx.x * 4 + quarter, 1u);
        }
        continue;
      }
      const float4* part = nullptr;   // TAIL: the previous pair's partial sums for these rows
      if (sg.kind == SEG_TAIL) {
        const int wslot = static_cast<int>(blockIdx.x) - 2;
        int fok = 1;
        if (lane == 0) fok = flag_wait(p.sk_flags + wslot * 4 + quarter, abort_flag, QLORA_DEV_TIMEOUT_EPI) ? 1 : 0;
        if (!__shfl_sync(0xFFFFFFFFu, fok, 0)) break;
        part = reinterpret_cast<const float4*>(p.sk_part + static_cast<size_t>(wslot) * (128 * TILE_COLS)) + prow;
      }
      if (p.tma_out) {
        // tensor memory column c: token group c / 256, feature c % 256
        auto pack = [&](const uint32_t (&r)[32], uint32_t (&pk)[16]) {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
        };
        // stage one converted 32 x 32 chunk in this warp's box and store it;
        // a chunk half inside the tile (FN % 32 == 16) goes out as two
        // 16-byte stores per row, a chunk past it not at all
        auto emit = [&](int ch, const uint32_t (&pk)[16]) {
          const int valid = FN - (ch % 8) * 32;
          if (valid < 32) {
            const int token = tile_tok(tile) + 256 * (ch / 8) + 128 * static_cast<int>(rank) + quarter * 32 + lane;
            const int fc = f0 + (ch % 8) * 32;
            if (valid > 0 && token < p.cols) {
              __nv_bfloat16* orow = out + static_cast<int64_t>(token) * p.ldo + fc;
              if (fc + 16 <= p.rows) {
                reinterpret_cast<uint4*>(orow)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                reinterpret_cast<uint4*>(orow)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
              } else {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                  if (fc + i < p.rows)
                    reinterpret_cast<uint16_t*>(orow)[i] = static_cast<uint16_t>(pk[i >> 1] >> (16 * (i & 1)));
              }
            }
            return;
          }
          if (lane == 0) bulk_wait_read_all();   // the previous store has read the box
          __syncwarp();
          const uint32_t row = box + lane * 64;
          const uint32_t sw = (lane >> 1) & 3;
#pragma unroll
          for (int v = 0; v < 4; ++v)
            sts128(row + ((v ^ sw) << 4), pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int h = ch / 8;
            const int token0 = tile_tok(tile) + 256 * h + 128 * static_cast<int>(rank) + quarter * 32;
            tma_store_2d(&tm_out, box, f0 + (ch % 8) * 32, token0);
            bulk_commit();
          }
        };
        if (part == nullptr) {
          // chunk ch + 1 loads from tensor memory while chunk ch is staged
          uint32_t ra[32], rb[32];
          tmem_ld_32x32b_x32(tbase, ra);
          tc_wait_ld();
#pragma unroll 1
          for (int ch = 0; ch < NCH; ch += 2) {
            {
              uint32_t pk[16];
              pack(ra, pk);
              tmem_ld_32x32b_x32(tbase + (ch + 1) * 32, rb);
              emit(ch, pk);
              tc_wait_ld();
            }
            {
              uint32_t pk[16];
              pack(rb, pk);
              if (ch + 2 < NCH) tmem_ld_32x32b_x32(tbase + (ch + 2) * 32, ra);
              emit(ch + 1, pk);
              if (ch + 2 < NCH) tc_wait_ld();
            }
          }
        } else {
          // TAIL: the partial sums are read two chunks ahead (they come from
          // L2 or HBM); one tensor-memory buffer keeps the registers in bounds
          float4 pa[8], pb[8];
          auto load_part = [&](int ch, float4 (&pq)[8]) {
#pragma unroll
            for (int v = 0; v < 8; ++v) pq[v] = __ldcg(part + (ch * 8 + v) * 128);
          };
          auto tail_chunk = [&](int ch, float4 (&pq)[8]) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tbase + ch * 32, r);
            tc_wait_ld();
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              r[4 * v] = __float_as_uint(__uint_as_float(r[4 * v]) + pq[v].x);
              r[4 * v + 1] = __float_as_uint(__uint_as_float(r[4 * v + 1]) + pq[v].y);
              r[4 * v + 2] = __float_as_uint(__uint_as_float(r[4 * v + 2]) + pq[v].z);
              r[4 * v + 3] = __float_as_uint(__uint_as_float(r[4 * v + 3]) + pq[v].w);
            }
            if (ch + 2 < NCH) load_part(ch + 2, pq);
            uint32_t pk[16];
            pack(r, pk);
            emit(ch, pk);
          };
          load_part(0, pa);
          load_part(1, pb);
#pragma unroll 1
          for (int ch = 0; ch < NCH; ch += 2) {
            tail_chunk(ch, pa);
            tail_chunk(ch + 1, pb);
          }
        }
        // every column of this accumulator has been read: release it now
        release_acc();
      } else {
#pragma unroll 1
        for (int h = 0; h < NH; ++h) {
          const int token = tile_tok(tile) + 256 * h + 128 * static_cast<int>(rank) + quarter * 32 + lane;
          __nv_bfloat16* orow = out + static_cast<int64_t>(token) * p.ldo;
          const uint32_t taddr = tbase + h * 256;
#pragma unroll 1
          for (int ch = 0; ch < 8; ch += 2) {
            uint32_t r0[32], r1[32];
            tmem_ld_32x32b_x32(taddr + ch * 32, r0);
            tmem_ld_32x32b_x32(taddr + ch * 32 + 32, r1);
            tc_wait_ld();
            if (token < p.cols) {
              const int lim = min(p.rows, f0 + FN);   // features of this tile
#pragma unroll
              for (int half = 0; half < 2; ++half) {
                const uint32_t* rr = half ? r1 : r0;
                const int fc = f0 + (ch + half) * 32;
                if (vec_ok && fc + 32 <= lim) {
                  uint4* dst = reinterpret_cast<uint4*>(orow + fc);
#pragma unroll
                  for (int v = 0; v < 4; ++v) {
                    dst[v] = make_uint4(pack_bf16x2(__uint_as_float(rr[8 * v + 0]), __uint_as_float(rr[8 * v + 1])),
                                        pack_bf16x2(__uint_as_float(rr[8 * v + 2]), __uint_as_float(rr[8 * v + 3])),
                                        pack_bf16x2(__uint_as_float(rr[8 * v + 4]), __uint_as_float(rr[8 * v + 5])),
                                        pack_bf16x2(__uint_as_float(rr[8 * v + 6]), __uint_as_float(rr[8 * v + 7])));
                  }
                } else {
#pragma unroll
                  for (int i = 0; i < 32; ++i)
                    if (fc + i < lim) orow[fc + i] = __float2bfloat16_rn(__uint_as_float(rr[i]));
                }
              }
            }
          }
        }
        release_acc();
      }
    }
    if (lane == 0) bulk_wait_all();   // stores complete before the CTA's shared memory goes away
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // no CTA leaves while its pair still reads its shared or tensor memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_ALLOC);
  }
}

#define QLORA_PAIR_INST(AS, NH)                                                                         \
  template __global__ void k_tc_pair<AS, NH>(const __grid_constant__ CUtensorMap,                       \
                                             const __grid_constant__ CUtensorMap,                       \
                                             const __grid_constant__ CUtensorMap,                       \
                                             const __grid_constant__ CUtensorMap, TcParams);
QLORA_PAIR_INST(A_DQ_K, 1)
QLORA_PAIR_INST(A_DQ_K, 2)
QLORA_PAIR_INST(A_DQ_MN, 1)
QLORA_PAIR_INST(A_DQ_MN, 2)

}  // namespace qlora
