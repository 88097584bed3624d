// Persistent, warp-specialised tcgen05 GEMM for sm_100a, grouped along M only.
//
// The expert FFN of an MoE layer is a set of independent GEMMs, one per expert, over a
// ragged number of token rows (routing primer "MoE 路由入门" §5.2; the "MoE" chapter
// index describes the grouped GEMM as grouping only the M axis with a contiguous
// layout).  Here the rows of all experts sit in one matrix A, each expert's bucket
// starting at a multiple of BM = 128, so every 128-row M-tile belongs to exactly one
// expert and the weights of that expert are the B operand.
//
//   out[r, n] = epilogue( sum_k A[r, k] * B[g*b_rows + n, k] )   for rows r of group g
//
// One CTA per SM walks a static list of uniform-cost work items (expert, N-tile,
// M-tile[, K-slice]), ordered expert by expert and, inside an expert, N-tile by N-tile with the
// expert's M-tiles adjacent: the CTAs running at the same time share each weight tile
// through L2, and an expert's activation rows stay L2-resident while its N-tiles run.
// Because all items cost the same, a skewed expert load does not leave a tail.
//
// Warp roles (192 threads):
//   warp 0     TMA producer: A tile (128 x 64) and B tile (BN x 64) per K-step into a
//              STAGES-deep ring of 128-byte-swizzled shared-memory stages
//   warp 1     TMEM allocator + UMMA issuer: 128 x BN x 16 tcgen05.mma, fp32 accumulator
//              in TMEM, two accumulators so the epilogue of one tile overlaps the
//              mainloop of the next
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//              32*(w%4)..+31), then one of
//                EPI_BF16   round to bf16 and store
//                EPI_SWIGLU B holds [gate rows; up rows] of the same output columns;
//                           h = SiLU(gate) * up, rounded to bf16
//                EPI_F32    store fp32 (router logits, down-projection outputs),
//                           columns >= N dropped
//                EPI_COMBINE down projection fused with the combine: each row r of a
//                           bucket is pair p = pair_of_row[r] of token t = p / K, and
//                           w[p] * y[r] is added to the fp32 token accumulator
//                           acc[t] with vector reductions (order of the K additions,
//                           and so the last bits, vary from run to run)
//
// Every wait on an mbarrier is bounded; on timeout the CTA sets MOE_DEV_TIMEOUT in the
// status word, drains the copies and MMAs it issued, frees TMEM and exits.
#pragma once

#include "common.cuh"

namespace moe {

enum EpiKind { EPI_BF16 = 0, EPI_SWIGLU = 1, EPI_F32 = 2, EPI_COMBINE = 3 };

struct GemmParams {
  const int32_t* offsets;  // [G+1] first row of each group (multiples of 128); nullptr: dense
  const int32_t* counts;   // [G] real rows of each group; rows past it (padding) are not
                           // stored.  nullptr: every row of a group's tiles is stored
  int G;                   // groups
  int dense_rows;          // rows of the single group when offsets == nullptr
  int K;                   // reduction length, multiple of 64
  int N;                   // output columns of one group
  int b_rows_per_group;    // rows of one group in the stacked B tensor map(s)
  void* out;               // [rows, ldo] bf16 or fp32
  int64_t ldo;             // leading dimension of out, in elements
  int32_t* status;         // device status word (may be null)
  const int32_t* pair_of_row;  // EPI_COMBINE: pair of each bucket row
  const float* pair_weight;    // EPI_COMBINE: combine weight of each pair [T*K]
  int topk;                    // EPI_COMBINE: K (pair p belongs to token p / K)
  int masked_cap;              // > 0: masked layout.  offsets is then only the schedule (the
                               // compact 128-padded prefix of counts); group g's rows sit at
                               // g * masked_cap in A and out
  int k_splits;                // > 1 (EPI_F32 only): the K loop of every tile is cut into
                               // k_splits slices, slice s adding K-blocks
                               // [s*KB/k_splits, (s+1)*KB/k_splits) into its own output
  long long split_stride;      // elements between the outputs of consecutive slices
  int half_tiles;              // 1 (grouped, with counts): an M-tile holding at most 64 real
                               // rows runs M=64 MMAs over its first 64 rows
};

// K-blocks [kb0, kb1) of slice `split` out of `splits` over KB K-blocks.
MOE_DEVINL void k_slice(int split, int splits, int KB, int& kb0, int& kb1) {
  kb0 = static_cast<int>(static_cast<long long>(split) * KB / splits);
  kb1 = static_cast<int>(static_cast<long long>(split + 1) * KB / splits);
}

MOE_DEVINL void red_add_v4(float* addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d, float w) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(w * __uint_as_float(a)),
               "f"(w * __uint_as_float(b)), "f"(w * __uint_as_float(c)), "f"(w * __uint_as_float(d))
               : "memory");
}

template <int BN_, int EPI_, int STAGES_>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BN = BN_;
  static constexpr int BK = 64;  // 64 bf16 = 128 bytes = one swizzle row
  static constexpr int EPI = EPI_;
  static constexpr int STAGES = STAGES_;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;  // + 1 KB alignment slack
  static constexpr int OUT_COLS = EPI == EPI_SWIGLU ? BN / 2 : BN;  // output columns per tile
  static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64
                                   : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
  static constexpr int ACC_COLS = TMEM_COLS / 2;                    // TMEM columns per accumulator
  static constexpr int THREADS = 192;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
  static_assert(EPI != EPI_SWIGLU || BN % 64 == 0, "SwiGLU tile holds gate and up halves");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

struct TileCoord {
  int m_tile;  // position in the schedule
  int n_tile;
  int group;
  int local0;  // first row of the tile inside its group
  int row0;    // first row of the tile in A and out
};

// Work item -> (M-tile, N-tile, group).  Items of group g occupy [mt0*NT, mt1*NT) where
// [mt0, mt1) are g's M-tiles.  Inside that range the operand with fewer rows is the one
// re-read from L2 by the CTAs running side by side: N-tiles outer (each weight tile is
// shared by all M-tiles in flight) when the group's weight rows NT*b_rows outnumber its
// activation rows, M-tiles outer (each activation tile shared by all N-tiles) otherwise,
// as for a hot expert of a skewed load or the dense shared expert.
MOE_DEVINL TileCoord decode_item(int item, int NT, const GemmParams& p, int num_m_tiles, int b_rows) {
  const int v = item / NT;  // an M-tile of the same group
  int g = 0, mt0 = 0, cnt = num_m_tiles;
  if (p.offsets != nullptr) {
    const int row = v * 128;
    int lo = 0, hi = p.G - 1;  // smallest g with offsets[g+1] > row
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(p.offsets + mid + 1) > row) hi = mid; else lo = mid + 1;
    }
    g = lo;
    mt0 = __ldg(p.offsets + g) >> 7;
    cnt = (__ldg(p.offsets + g + 1) >> 7) - mt0;
  }
  const int local = item - mt0 * NT;
  const bool m_outer = cnt * 128 > NT * b_rows;
  TileCoord t;
  t.m_tile = mt0 + (m_outer ? local / NT : local % cnt);
  t.n_tile = m_outer ? local % NT : local / cnt;
  t.group = g;
  t.local0 = (t.m_tile - mt0) * 128;
  t.row0 = p.masked_cap > 0 ? g * p.masked_cap + t.local0 : t.m_tile * 128;
  return t;
}

// Whether tile t runs M=64 MMAs: its group has at most 64 real rows from the tile's first
// row on.  The M=64 accumulator of a one-SM MMA holds tile row 16i + j in TMEM lane
// 32i + j (j < 16): lanes 0-15 of each 32-lane quadrant.
MOE_DEVINL bool half_tile(const TileCoord& t, const GemmParams& p) {
  return p.half_tiles && p.offsets != nullptr && p.counts != nullptr &&
         __ldg(p.counts + t.group) - t.local0 <= 64;
}

MOE_DEVINL float silu_mul(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                   const __grid_constant__ CUtensorMap tmB1, const GemmParams p) {
  constexpr int BM = Cfg::BM, BN = Cfg::BN, BK = Cfg::BK, STAGES = Cfg::STAGES;
  constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);

  extern __shared__ uint8_t dsmem[];
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ uint64_t tfull_bar[2], tempty_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = warp_id(), lane = lane_id();
  const uint32_t pad = (1024u - (smem_u32(dsmem) & 1023u)) & 1023u;
  uint8_t* smem = dsmem + pad;

  const int NT = (p.N + Cfg::OUT_COLS - 1) / Cfg::OUT_COLS;
  const int KB = p.K / BK;
  const int S = p.k_splits > 1 ? p.k_splits : 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 128);
    }
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB0);
    if (Cfg::EPI == EPI_SWIGLU) prefetch_tmap(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  // the offsets (and A) come from the kernels before this one
  pdl_launch_dependents();
  pdl_wait();
  const int num_m_tiles = p.offsets ? (__ldg(p.offsets + p.G) >> 7) : (p.dense_rows + BM - 1) / BM;
  const int total = num_m_tiles * NT * S;  // CTAs past it run no item

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const TileCoord t = decode_item(item / S, NT, p, num_m_tiles, BN);
        int kb0, kb1;
        k_slice(item % S, S, KB, kb0, kb1);
        const int a_row = t.row0;
        const int b_row = t.group * p.b_rows_per_group + t.n_tile * Cfg::OUT_COLS;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, &abort_flag)) { ok = false; break; }
          uint8_t* sa = smem + s * Cfg::STAGE_BYTES;
          uint8_t* sb = sa + Cfg::A_BYTES;
          mbar_arrive_expect_tx(&full_bar[s], Cfg::STAGE_BYTES);
          tma_load_2d(sa, &tmA, kb * BK, a_row, &full_bar[s]);
          if (Cfg::EPI == EPI_SWIGLU) {
            tma_load_2d(sb, &tmB0, kb * BK, b_row, &full_bar[s]);
            tma_load_2d(sb + (BN / 2) * BK * 2, &tmB1, kb * BK, b_row, &full_bar[s]);
          } else {
            tma_load_2d(sb, &tmB0, kb * BK, b_row, &full_bar[s]);
          }
          ++issued;
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      // Wait until the last loads this thread issued have landed (they have, unless the
      // pipeline was aborted), so no copy is in flight when the CTA exits.
      volatile int no_abort = 0;
      const long long back = issued < STAGES ? issued : STAGES;
      for (long long j = 0; j < back; ++j) {
        if (s == 0) { s = STAGES - 1; ph ^= 1u; } else { --s; }
        mbar_wait_bounded(&full_bar[s], ph, &no_abort);
      }
      if (!ok || no_abort) abort_flag = 1;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- UMMA issuer
    if (lane == 0) {
      int s = 0, acc = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
        if (!mbar_wait_bounded(&tempty_bar[acc], acc_ph ^ 1u, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * Cfg::ACC_COLS;
        int kb0, kb1;
        k_slice(item % S, S, KB, kb0, kb1);
        const uint32_t idesc = half_tile(decode_item(item / S, NT, p, num_m_tiles, BN), p)
                                   ? idesc_bf16_f32(64, BN) : IDESC;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint32_t b0 = a0 + Cfg::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            umma_f16(d_tmem, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), idesc,
                     (kb != kb0) || (k != 0));
          }
          umma_commit(&empty_bar[s]);  // frees the stage once these MMAs have read it
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);  // accumulator ready for the epilogue
        if (++acc == 2) { acc = 0; acc_ph ^= 1u; }
      }
      // Every MMA issued above has completed once drain_bar flips.
      umma_commit(&drain_bar);
      volatile int no_abort = 0;
      mbar_wait_bounded(&drain_bar, 0, &no_abort);
      if (!ok || no_abort) abort_flag = 1;
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      const TileCoord t = decode_item(item / S, NT, p, num_m_tiles, BN);
      // every lane polls, then the warp agrees (tcgen05.ld below is warp-collective)
      const bool ready = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull_bar[acc], acc_ph, &abort_flag));
      if (!ready) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * Cfg::ACC_COLS;
      const bool half = half_tile(t, p);
      const int trow = half ? q * 16 + lane : q * 32 + lane;  // tile row held by this lane
      const long long row = static_cast<long long>(t.row0) + trow;
      bool row_ok;
      if (p.offsets == nullptr) row_ok = row < p.dense_rows;
      else if (p.counts == nullptr) row_ok = true;
      else row_ok = (!half || lane < 16) && t.local0 + trow < __ldg(p.counts + t.group);
      const int col0 = t.n_tile * Cfg::OUT_COLS;

      if constexpr (Cfg::EPI == EPI_SWIGLU) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + row * p.ldo + col0;
        const bool v8 = ((reinterpret_cast<uintptr_t>(p.out) | (static_cast<uintptr_t>(p.ldo) * 2)) & 31) == 0;
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t rg[32], ru[32];
          tmem_ld_32x32b_x32(tbase + c, rg);
          tmem_ld_32x32b_x32(tbase + BN / 2 + c, ru);
          tmem_ld_wait(rg);
          reg_fence(ru);
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float h0 = silu_mul(__uint_as_float(rg[2 * i]), __uint_as_float(ru[2 * i]));
            const float h1 = silu_mul(__uint_as_float(rg[2 * i + 1]), __uint_as_float(ru[2 * i + 1]));
            packed[i] = pack_bf16x2(h0, h1);
          }
          if (row_ok && col0 + c < p.N) {
            if (v8) {
              st_global_v8(out + c, packed);
              st_global_v8(out + c + 16, packed + 8);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
              for (int v = 0; v < 4; ++v)
                dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
            }
          }
        }
      } else if constexpr (Cfg::EPI == EPI_COMBINE) {
        int pair = -1;
        if (row_ok) pair = __ldg(p.pair_of_row + row);
        const float wgt = pair >= 0 ? __ldg(p.pair_weight + pair) : 0.f;
        float* out = static_cast<float*>(p.out) + static_cast<long long>(pair >= 0 ? pair / p.topk : 0) * p.ldo + col0;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + c, r);
          tmem_ld_wait(r);
          if (pair >= 0 && col0 + c < p.N) {
#pragma unroll
            for (int v = 0; v < 8; ++v) red_add_v4(out + c + 4 * v, r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3], wgt);
          }
        }
      } else if constexpr (Cfg::EPI == EPI_BF16) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + row * p.ldo + col0;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + c, r);
          tmem_ld_wait(r);
          if (row_ok && col0 + c < p.N) {
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              packed[i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
            uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
          }
        }
      } else if constexpr (BN % 32 == 0) {
        float* out = static_cast<float*>(p.out) + (item % S) * p.split_stride + row * p.ldo + col0;
        const bool v8 = ((reinterpret_cast<uintptr_t>(p.out) | (static_cast<uintptr_t>(p.ldo) * 4)) & 31) == 0;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + c, r);
          tmem_ld_wait(r);
          if (row_ok) {
            if (v8 && col0 + c + 32 <= p.N) {
#pragma unroll
              for (int v = 0; v < 4; ++v) st_global_v8(out + c + 8 * v, r + 8 * v);
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (col0 + c + i < p.N) out[c + i] = __uint_as_float(r[i]);
            }
          }
        }
      } else {
        float* out = static_cast<float*>(p.out) + (item % S) * p.split_stride + row * p.ldo + col0;
#pragma unroll 1
        for (int c = 0; c < BN; c += 16) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(tbase + c, r);
          tmem_ld_wait(r);
          if (row_ok) {
            if (col0 + c + 16 <= p.N && (p.ldo & 3) == 0) {
              uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
              for (int v = 0; v < 4; ++v) dst[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (col0 + c + i < p.N) out[c + i] = __uint_as_float(r[i]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);
      if (++acc == 2) { acc = 0; acc_ph ^= 1u; }
    }
  }

  __syncthreads();
  if (abort_flag && threadIdx.x == 0) set_status(p.status, MOE_DEV_TIMEOUT);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace moe
