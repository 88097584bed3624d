// Grouped expert GEMMs with two M-tiles per work item: the gate/up projection with fused
// SwiGLU (SWIGLU = true) and the down projection (fp32 or fp16 out).  With no schedule
// (offsets == nullptr) the A rows form one dense group, as for the shared expert.  With
// x_rows > 0 a dense extra group follows the G groups in the same launch, with A, weights
// and output of its own (tmA2 / tmG2 / tmU2, x_out): the shared expert of a layer whose
// routed experts also take two M-tiles per item, so the two share one launch and one tail.
//
// The same grouped GEMMs as tc_gemm_kernel<EPI_SWIGLU / EPI_F32> (routing primer "MoE 路由入门"
// §5.2; the "MoE" chapter index's M-grouped contiguous layout), with one change in how a
// CTA spends its shared memory: a work item is up to two consecutive 128-row M-tiles of one
// expert against one 256-row weight tile ([128 gate rows; 128 up rows], or 256 rows of
// W_down).  Each K-step stage
// holds both A tiles and the one B tile (64 KB), and the MMA thread issues, per 16-wide K
// slice, one M=128 N=256 tcgen05.mma per M-tile into its own 256-column TMEM accumulator.
// Every weight tile staged in shared memory is so used twice, which halves the weight
// bytes moved from L2 per FLOP.  An expert with an odd number of M-tiles ends with a
// one-tile item.
//
// Items cost one or two tile-units, so a static split would leave CTAs idle at the end.
// The producer warp takes items in order from a global counter (atomicAdd on a word the
// host zeroes before the launch) and passes each to the MMA thread and the epilogue warps
// through a small ring in shared memory; items of one (expert, weight tile) still start
// side by side on different CTAs, so the weight tile crosses HBM once.
//
// TMEM: two 256-column accumulators (slots).  A two-tile item uses both, a one-tile item
// the next free one; the epilogue releases a slot as soon as it has read it.  A tile with
// at most 64 real rows runs M=64 MMAs (accumulator rows in lanes 0-15 of each quadrant).
//
// Warp roles (192 threads): warp 0 takes items and issues TMA loads, warp 1 allocates
// TMEM and issues MMAs, warps 2-5 run the epilogue.  Every wait is bounded; on a
// timeout the CTA sets MOE_DEV_TIMEOUT, drains its copies and MMAs, frees TMEM and exits.
#pragma once

#include "tc_gemm.cuh"

namespace moe {

struct DualParams {
  const int32_t* offsets;   // [G+1] schedule: first row of each group, multiples of 128;
                            // nullptr: one dense group of dense_rows rows (G = 1)
  const int32_t* counts;    // [G] real rows of each group (rows past it are not stored)
  int dense_rows;
  int G;                    // groups (G <= kDualMaxGroups)
  int K;                    // reduction length, multiple of 64
  int N;                    // output columns; weight rows per group (and matrix, for SwiGLU)
  int masked_cap;           // > 0: group g's rows sit at g * masked_cap in A and out
  void* out;                // SwiGLU: h [rows, ldo] bf16; else y [rows, ldo] fp32 (fp16: out_f16)
  int64_t ldo;
  int32_t* status;
  int32_t* next_item;       // work counter, zero at launch
  int out_f16;              // plain projection: store y as fp16 (|y| > 65504 sets MOE_DEV_RANGE)
  // the extra dense group (0 rows: none): its rows, output columns, reduction length
  // (multiple of 64) and output, stored like the others (out_f16 applies to it as well)
  int x_rows, x_N, x_K;
  void* x_out;
  int64_t x_ldo;
};

constexpr int kDualMaxGroups = 1024;
constexpr int kDualStages = 3;
constexpr int kDualBK = 64;
constexpr int kDualABytes = 128 * kDualBK * 2;                 // one M-tile's K-step
constexpr int kDualBBytes = 256 * kDualBK * 2;                 // gate + up rows
constexpr int kDualStageBytes = 2 * kDualABytes + kDualBBytes;  // 64 KB
constexpr int kDualSmemBytes = kDualStages * kDualStageBytes + 1024;
constexpr int kDualRing = 4;                                   // items between producer and consumers
constexpr int kDualThreads = 192;
static_assert(kDualSmemBytes + (kDualMaxGroups + 2) * 4 + 1024 <= 227 * 1024, "shared memory");

struct DualItem {
  int group;
  int n_tile;
  int tile0;     // first M-tile of the item, in the schedule
  int ntiles;    // 1 or 2
  int mt0;       // first M-tile of the group
};

// Item -> (group, weight tile, M-tiles); weight tiles of 128 output columns for SwiGLU
// (128 gate + 128 up rows), of 256 for the plain projection.  pref[g] = sum over e < g of NT * pairs(e), with
// pairs(e) = ceil(tiles(e) / 2).  Inside a group, weight tiles are outer (every pair of
// M-tiles in flight shares each weight tile) unless the group's activation rows outnumber
// its weight rows (NT * 256), as for a very hot expert, where pairs are outer.
// First row of group g in the schedule (g = G: the end), and its real rows.
MOE_DEVINL int group_row(const DualParams& p, int g) {
  return p.offsets != nullptr ? __ldg(p.offsets + g) : (g == 0 ? 0 : (p.dense_rows + 127) / 128 * 128);
}
MOE_DEVINL int group_count(const DualParams& p, int g) {
  return p.offsets != nullptr ? __ldg(p.counts + g) : p.dense_rows;
}

MOE_DEVINL DualItem dual_decode(int item, int NT, int NT2, const DualParams& p, const int* pref) {
  // (NT * 256 is the group's weight rows in both forms: SwiGLU tiles hold 256 rows too)
  if (item >= pref[p.G]) {  // the extra dense group (group index G)
    const int tiles = (p.x_rows + 127) >> 7;
    const int pairs = (tiles + 1) >> 1;
    const int local = item - pref[p.G];
    const bool pairs_outer = tiles * 128 > NT2 * 256;
    const int j = pairs_outer ? local / NT2 : local % pairs;
    DualItem d;
    d.group = p.G;
    d.n_tile = pairs_outer ? local % NT2 : local / pairs;
    d.tile0 = 2 * j;
    d.ntiles = (2 * j + 1 < tiles) ? 2 : 1;
    d.mt0 = 0;
    return d;
  }
  int lo = 0, hi = p.G - 1;  // group with pref[g] <= item < pref[g+1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pref[mid] <= item) lo = mid; else hi = mid - 1;
  }
  const int g = lo;
  const int mt0 = group_row(p, g) >> 7;
  const int tiles = (group_row(p, g + 1) >> 7) - mt0;
  const int pairs = (tiles + 1) >> 1;
  const int local = item - pref[g];
  const bool pairs_outer = tiles * 128 > NT * 256;
  const int j = pairs_outer ? local / NT : local % pairs;
  DualItem d;
  d.group = g;
  d.n_tile = pairs_outer ? local % NT : local / pairs;
  d.tile0 = mt0 + 2 * j;
  d.ntiles = (2 * j + 1 < tiles) ? 2 : 1;
  d.mt0 = mt0;
  return d;
}

// SWIGLU: tmG / tmU are the gate and up weights (boxes of 128 rows) and h = SiLU(g) * u is
// stored in bf16; otherwise tmG is the one weight matrix (boxes of 256 rows) and the
// product is stored in fp32, or in fp16 with out_f16.
template <bool SWIGLU>
__global__ void __launch_bounds__(kDualThreads, 1)
    tc_gemm_dual_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmG,
                        const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmA2,
                        const __grid_constant__ CUtensorMap tmG2, const __grid_constant__ CUtensorMap tmU2,
                        const DualParams p) {
  constexpr int OUT_COLS = SWIGLU ? 128 : 256;
  constexpr int BK = kDualBK, STAGES = kDualStages, R = kDualRing;
  constexpr uint32_t IDESC = idesc_bf16_f32(128, 256);
  constexpr uint32_t IDESC_HALF = idesc_bf16_f32(64, 256);

  extern __shared__ uint8_t dsmem[];
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ uint64_t tfull_bar[2], tempty_bar[2], drain_bar;
  __shared__ uint64_t item_full[R], item_empty[R];
  __shared__ int item_ring[R];
  __shared__ int pref[kDualMaxGroups + 2];
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;

  const int warp = warp_id(), lane = lane_id();
  const uint32_t pad = (1024u - (smem_u32(dsmem) & 1023u)) & 1023u;
  uint8_t* smem = dsmem + pad;
  const int NT = (p.N + OUT_COLS - 1) / OUT_COLS;
  const int NT2 = (p.x_N + OUT_COLS - 1) / OUT_COLS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 128);
    }
    for (int r = 0; r < R; ++r) {
      mbar_init(&item_full[r], 1);
      mbar_init(&item_empty[r], 5);  // the MMA thread and one lane of each epilogue warp
    }
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmG);
    if (SWIGLU) prefetch_tmap(&tmU);
    if (p.x_rows > 0) {
      prefetch_tmap(&tmA2);
      prefetch_tmap(&tmG2);
      if (SWIGLU) prefetch_tmap(&tmU2);
    }
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  // the schedule, counts and A come from the kernels before this one
  pdl_launch_dependents();
  pdl_wait();
  if (warp == 2) {
    // pref[g] over the groups, one warp: each lane sums a contiguous run, then a scan
    const int per = (p.G + 31) / 32;
    const int g0 = lane * per;
    int run = 0;
    for (int g = g0; g < g0 + per && g < p.G; ++g) {
      const int tiles = (group_row(p, g + 1) - group_row(p, g)) >> 7;
      run += NT * ((tiles + 1) >> 1);
    }
    int incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int acc = incl - run;
    for (int g = g0; g < g0 + per && g < p.G; ++g) {
      pref[g] = acc;
      const int tiles = (group_row(p, g + 1) - group_row(p, g)) >> 7;
      acc += NT * ((tiles + 1) >> 1);
    }
    if (lane == 31) {
      pref[p.G] = incl;
      const int x_tiles = (p.x_rows + 127) >> 7;
      pref[p.G + 1] = incl + (p.x_rows > 0 ? NT2 * ((x_tiles + 1) >> 1) : 0);
    }
  }
  __syncthreads();
  const int total = pref[p.G + 1];

  if (warp == 0) {
    // ---------------------------------------------------------------- scheduler + TMA
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int rs = i % R;
        const uint32_t rph = static_cast<uint32_t>(i / R) & 1u;
        if (!mbar_wait_bounded(&item_empty[rs], rph ^ 1u, &abort_flag)) { ok = false; break; }
        const int it = atomicAdd(p.next_item, 1);
        item_ring[rs] = it;
        mbar_arrive(&item_full[rs]);
        if (it >= total) break;
        const DualItem d = dual_decode(it, NT, NT2, p, pref);
        const bool ex = d.group == p.G;  // the extra dense group
        const CUtensorMap* mA = ex ? &tmA2 : &tmA;
        const CUtensorMap* mG = ex ? &tmG2 : &tmG;
        const CUtensorMap* mU = ex ? &tmU2 : &tmU;
        const int b_row = (ex ? 0 : d.group * p.N) + d.n_tile * OUT_COLS;
        // (scalars, not arrays: an array indexed at run time lives in local memory)
        const int local0 = (d.tile0 - d.mt0) * 128;
        const int a_row0 = (p.masked_cap > 0 && !ex) ? d.group * p.masked_cap + local0 : d.tile0 * 128;
        const int a_row1 = a_row0 + 128;
        const int KB = (ex ? p.x_K : p.K) / BK;
        const uint32_t tx = static_cast<uint32_t>(d.ntiles * kDualABytes + kDualBBytes);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, &abort_flag)) { ok = false; break; }
          uint8_t* st = smem + s * kDualStageBytes;
          mbar_arrive_expect_tx(&full_bar[s], tx);
          tma_load_2d(st, mA, kb * BK, a_row0, &full_bar[s]);
          if (d.ntiles == 2) tma_load_2d(st + kDualABytes, mA, kb * BK, a_row1, &full_bar[s]);
          tma_load_2d(st + 2 * kDualABytes, mG, kb * BK, b_row, &full_bar[s]);
          if (SWIGLU) tma_load_2d(st + 2 * kDualABytes + kDualBBytes / 2, mU, kb * BK, b_row, &full_bar[s]);
          ++issued;
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      volatile int no_abort = 0;
      const long long back = issued < STAGES ? issued : STAGES;
      for (long long j = 0; j < back; ++j) {
        if (s == 0) { s = STAGES - 1; ph ^= 1u; } else { --s; }
        mbar_wait_bounded(&full_bar[s], ph, &no_abort);
      }
      if (!ok || no_abort) abort_flag = 1;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0, nxt = 0;
      uint32_t ph = 0;
      uint32_t uses = 0u;  // bit a: phase of slot a's accumulator
      bool ok = true;
      for (int i = 0; ok; ++i) {
        const int rs = i % R;
        const uint32_t rph = static_cast<uint32_t>(i / R) & 1u;
        if (!mbar_wait_bounded(&item_full[rs], rph, &abort_flag)) { ok = false; break; }
        const int it = item_ring[rs];
        mbar_arrive(&item_empty[rs]);
        if (it >= total) break;
        const DualItem d = dual_decode(it, NT, NT2, p, pref);
        const bool ex = d.group == p.G;
        const int KB = (ex ? p.x_K : p.K) / BK;
        const int slot0 = nxt, slot1 = nxt ^ 1;
        if (d.ntiles == 1) nxt ^= 1;
        const int rows0 = (ex ? p.x_rows : group_count(p, d.group)) - (d.tile0 - d.mt0) * 128;
        const uint32_t idesc0 = rows0 <= 64 ? IDESC_HALF : IDESC;
        const uint32_t idesc1 = rows0 - 128 <= 64 ? IDESC_HALF : IDESC;
        if (!mbar_wait_bounded(&tempty_bar[slot0], ((uses >> slot0) & 1u) ^ 1u, &abort_flag)) { ok = false; break; }
        if (d.ntiles == 2 &&
            !mbar_wait_bounded(&tempty_bar[slot1], ((uses >> slot1) & 1u) ^ 1u, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d0 = tmem_base + slot0 * 256, d1 = tmem_base + slot1 * 256;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * kDualStageBytes);
          const uint32_t a1 = a0 + kDualABytes;
          const uint32_t b0 = a0 + 2 * kDualABytes;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint32_t acc = (kb | k) != 0;
            umma_f16(d0, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), idesc0, acc);
            if (d.ntiles == 2) umma_f16(d1, smem_desc_sw128(a1 + k * 32), smem_desc_sw128(b0 + k * 32), idesc1, acc);
          }
          umma_commit(&empty_bar[s]);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[slot0]);
        uses ^= 1u << slot0;
        if (d.ntiles == 2) {
          umma_commit(&tfull_bar[slot1]);
          uses ^= 1u << slot1;
        }
      }
      umma_commit(&drain_bar);
      volatile int no_abort = 0;
      mbar_wait_bounded(&drain_bar, 0, &no_abort);
      if (!ok || no_abort) abort_flag = 1;
    }
  } else {
    // ---------------------------------------------------------------- SwiGLU epilogue
    const int q = warp & 3;
    int nxt = 0;
    uint32_t uses = 0u;  // bit a: phase of slot a's accumulator
    const bool v8_main = ((reinterpret_cast<uintptr_t>(p.out) | (static_cast<uintptr_t>(p.ldo) * (SWIGLU ? 2 : 4))) & 31) == 0;
    const bool v8_x = ((reinterpret_cast<uintptr_t>(p.x_out) | (static_cast<uintptr_t>(p.x_ldo) * (SWIGLU ? 2 : 4))) & 31) == 0;
    bool ok = true;
    for (int i = 0; ok; ++i) {
      const int rs = i % R;
      const uint32_t rph = static_cast<uint32_t>(i / R) & 1u;
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&item_full[rs], rph, &abort_flag));
      if (!ok) break;
      const int it = item_ring[rs];
      __syncwarp();
      if (lane == 0) mbar_arrive(&item_empty[rs]);
      if (it >= total) break;
      const DualItem d = dual_decode(it, NT, NT2, p, pref);
      const bool ex = d.group == p.G;
      const int slot0 = nxt, slot1 = nxt ^ 1;
      if (d.ntiles == 1) nxt ^= 1;
      const int count = ex ? p.x_rows : group_count(p, d.group);
      const int col0 = d.n_tile * OUT_COLS;
      const int n_cols = ex ? p.x_N : p.N;
      void* const out_base = ex ? p.x_out : p.out;
      const int64_t ldo = ex ? p.x_ldo : p.ldo;
      const bool v8 = ex ? v8_x : v8_main;
      for (int u = 0; u < d.ntiles && ok; ++u) {
        const int slot = u == 0 ? slot0 : slot1;
        ok = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull_bar[slot], (uses >> slot) & 1u, &abort_flag));
        if (!ok) break;
        tc_fence_after();
        const int local0 = (d.tile0 + u - d.mt0) * 128;
        const int row0 = (p.masked_cap > 0 && !ex) ? d.group * p.masked_cap + local0 : (d.tile0 + u) * 128;
        const bool half = count - local0 <= 64;
        const int trow = half ? q * 16 + lane : q * 32 + lane;
        const bool row_ok = (!half || lane < 16) && local0 + trow < count;
        const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + slot * 256;
        const long long orow = static_cast<long long>(row0) + trow;
        if constexpr (SWIGLU) {
          __nv_bfloat16* out = static_cast<__nv_bfloat16*>(out_base) + orow * ldo + col0;
#pragma unroll 1
          for (int c = 0; c < 128; c += 32) {
            uint32_t rg[32], ru[32];
            tmem_ld_32x32b_x32(tbase + c, rg);
            tmem_ld_32x32b_x32(tbase + 128 + c, ru);
            tmem_ld_wait(rg);
            reg_fence(ru);
            uint32_t packed[16];
#pragma unroll
            for (int e = 0; e < 16; ++e)
              packed[e] = pack_bf16x2(silu_mul(__uint_as_float(rg[2 * e]), __uint_as_float(ru[2 * e])),
                                      silu_mul(__uint_as_float(rg[2 * e + 1]), __uint_as_float(ru[2 * e + 1])));
            if (row_ok && col0 + c < n_cols) {
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
        } else if (p.out_f16) {
          __half* out = static_cast<__half*>(out_base) + orow * ldo + col0;
          bool range_ok = true;
#pragma unroll 1
          for (int c = 0; c < 256; c += 32) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tbase + c, r);
            tmem_ld_wait(r);
            if (row_ok && col0 + c < n_cols) {
              uint32_t packed[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const float a = __uint_as_float(r[2 * e]), b = __uint_as_float(r[2 * e + 1]);
                range_ok = range_ok && fabsf(a) <= 65504.f && fabsf(b) <= 65504.f;
                __half2 hv = __floats2half2_rn(a, b);
                packed[e] = *reinterpret_cast<uint32_t*>(&hv);
              }
              st_global_v8(out + c, packed);
              st_global_v8(out + c + 16, packed + 8);
            }
          }
          if (!range_ok) set_status(p.status, MOE_DEV_RANGE);
        } else {
          float* out = static_cast<float*>(out_base) + orow * ldo + col0;
#pragma unroll 1
          for (int c = 0; c < 256; c += 32) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tbase + c, r);
            tmem_ld_wait(r);
            if (row_ok && col0 + c < n_cols) {
              if (v8 && col0 + c + 32 <= n_cols) {
#pragma unroll
                for (int v = 0; v < 4; ++v) st_global_v8(out + c + 8 * v, r + 8 * v);
              } else {
#pragma unroll
                for (int e = 0; e < 32; ++e)
                  if (col0 + c + e < n_cols) out[c + e] = __uint_as_float(r[e]);
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty_bar[slot]);
        uses ^= 1u << slot;
      }
    }
  }

  __syncthreads();
  if (abort_flag && threadIdx.x == 0) set_status(p.status, MOE_DEV_TIMEOUT);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace moe
