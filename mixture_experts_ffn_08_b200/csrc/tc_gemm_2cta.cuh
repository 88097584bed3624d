// Two-SM (tcgen05 cta_group::2) variant of the persistent grouped GEMM for sm_100a.
//
// A cluster of two CTAs on two SMs computes one 256 x BN tile with a single stream of
// UMMA instructions (M = 256): each CTA holds 128 rows of A and half of the BN rows of B
// in its shared memory, and its TMEM receives the accumulator of its own 128 rows.  Each
// B byte therefore crosses L2 -> SM once per 256 output rows instead of once per 128, the
// SM-side traffic per FLOP drops by a third, and the tensor core sees the same operand
// tile twice as long.  Buckets must start at multiples of 256 rows (block_m = 256) so
// both M-tiles of a pair belong to the same expert.
//
// Roles per CTA (192 threads), rank 0 of the pair is the leader:
//   warp 0     TMA producer in both CTAs: own A rows, own half of B (and, for FP8, the
//              own A scale atom plus all B scale atoms) into its own stage ring; the
//              copies complete on the LEADER's stage barrier (.cta_group::2 form), whose
//              expected byte count covers both CTAs
//   warp 1     TMEM allocation in both CTAs (cta_group::2); in the leader, the single
//              thread that issues tcgen05.mma.cta_group::2 and the commits, multicast to
//              both CTAs' "stage free" and "accumulator full" barriers
//   warps 2-5  epilogue in both CTAs on their own TMEM lanes; each warp signals the
//              leader's "accumulator free" barrier remotely
// Cluster barriers are used only at start (barriers initialised, TMEM allocated) and at
// the end (everything drained), which every thread reaches because every wait in
// between is bounded.  No multicast copies are used.
#pragma once

#include "tc_gemm_fp8.cuh"

namespace moe {

// ------------------------------------------------------------------ cluster helpers
MOE_DEVINL uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Shared::cluster address of the variable at `local` in CTA `rank` of the cluster.
MOE_DEVINL uint32_t mapa_shared(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

MOE_DEVINL void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

MOE_DEVINL void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// 2D TMA load into this CTA's shared memory whose completion is counted on the barrier
// at `bar_cluster` (the leader CTA's), as a 2-SM pair requires.
MOE_DEVINL void tma_load_2d_pair(void* smem_dst, const CUtensorMap* m, int32_t c0, int32_t c1,
                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(c0), "r"(c1), "r"(bar_cluster)
      : "memory");
}

MOE_DEVINL void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
MOE_DEVINL void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
MOE_DEVINL void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

MOE_DEVINL void umma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

MOE_DEVINL void umma_mxf8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                               uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Scale atoms of both CTAs of the pair (each from its own shared memory) into each CTA's
// own TMEM at the same address.
MOE_DEVINL void tmem_cp_pair_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Arrives on this CTA's barrier once every pair MMA issued by this thread is done.
MOE_DEVINL void umma_commit_pair_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Arrives on the barrier at this offset in both CTAs once this thread's MMAs are done.
MOE_DEVINL void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(static_cast<uint16_t>(0x3))
      : "memory");
}

// ------------------------------------------------------------------ configuration
enum Epi2 { EPI2_SWIGLU_BF16 = 0, EPI2_SWIGLU_E4M3 = 1, EPI2_F32 = 2, EPI2_BF16 = 3 };

template <int BN_, int EPI_, int STAGES_, bool FP8_>
struct Pair2Cfg {
  static constexpr int BM = 128;                 // rows per CTA; the pair covers 256
  static constexpr int BN = BN_;                 // UMMA N (columns of the accumulator)
  static constexpr bool FP8 = FP8_;
  static constexpr int BK = FP8 ? 128 : 64;      // elements per stage row (128 bytes)
  static constexpr int EPI = EPI_;
  static constexpr int STAGES = STAGES_;
  static constexpr int A_BYTES = BM * 128;
  static constexpr int B_HALF = BN / 2;          // B rows held by each CTA
  static constexpr int B_BYTES = B_HALF * 128;
  static constexpr int SFB_ATOMS = FP8 ? BN / 128 : 0;
  static constexpr int SF_BYTES = FP8 ? 512 * (1 + SFB_ATOMS) : 0;
  static constexpr int CTA_TX = A_BYTES + B_BYTES + SF_BYTES;   // bytes one CTA loads per stage
  static constexpr int STAGE_BYTES = (CTA_TX + 1023) / 1024 * 1024;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
  static constexpr bool SWIGLU = EPI == EPI2_SWIGLU_BF16 || EPI == EPI2_SWIGLU_E4M3;
  static constexpr int OUT_COLS = SWIGLU ? BN / 2 : BN;
  static constexpr int SF_COLS = FP8 ? 4 + 4 * SFB_ATOMS : 0;
  static constexpr int ACC_STAGES = (2 * BN + SF_COLS <= 512) ? 2 : 1;
  static constexpr int ACC_COLS = BN;
  static constexpr int SF_COL = ACC_STAGES * ACC_COLS;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 192;
  static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "UMMA N for M=256");
  static_assert(!FP8 || BN % 128 == 0, "FP8: B rows in whole 128-row scale atoms");
  static_assert(!SWIGLU || BN == 256, "SwiGLU tile = 128 gate + 128 up rows, one half per CTA");
  static_assert(SF_COL + SF_COLS <= TMEM_COLS, "TMEM columns");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(EPI != EPI2_SWIGLU_E4M3 || FP8, "e4m3 h only on the FP8 path");
};

struct Pair2Params {
  const int32_t* offsets;  // [G+1] first row of each group, multiples of 256
  const int32_t* counts;   // [G] real rows (pad rows are not stored), or nullptr
  int G;
  int K;                   // reduction length (multiple of BK)
  int N;                   // output columns of one group
  void* out;
  int64_t ldo;
  uint8_t* out_sf;         // e4m3 h: scale atoms [m_tiles][N/128][512]
  int32_t* status;
};

struct PairTile {
  int m_tile;  // this CTA's 128-row tile
  int n_tile;
  int group;
};

// Work item -> (256-row pair, N-tile, group); items of group g cover its pairs times the
// N-tiles, N-tiles outer and pairs inner, groups in order.
MOE_DEVINL PairTile decode_pair_item(int item, int NT, const Pair2Params& p, int num_pairs, uint32_t rank) {
  const int v = item / NT;
  int lo = 0, hi = p.G - 1;
  const int row = v * 256;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(p.offsets + mid + 1) > row) hi = mid; else lo = mid + 1;
  }
  const int pt0 = __ldg(p.offsets + lo) >> 8;
  const int cnt = (__ldg(p.offsets + lo + 1) >> 8) - pt0;
  const int local = item - pt0 * NT;
  PairTile t;
  t.m_tile = 2 * (pt0 + local % cnt) + static_cast<int>(rank);
  t.n_tile = local / cnt;
  t.group = lo;
  (void)num_pairs;
  return t;
}

// tmB0 / tmB1: weight maps (SwiGLU: gate for rank 0, up for rank 1; else one map used
// by both ranks).  FP8: tmSfa over A scale atoms, tmSfb0/1 over weight scale atoms
// (2D views [atoms, 128] of 32-bit words).
template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmSfa,
                        const __grid_constant__ CUtensorMap tmSfb0, const __grid_constant__ CUtensorMap tmSfb1,
                        const Pair2Params p) {
  constexpr int BN = Cfg::BN, BK = Cfg::BK, STAGES = Cfg::STAGES, ACC_STAGES = Cfg::ACC_STAGES;

  extern __shared__ uint8_t dsmem[];
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ uint64_t tfull_bar[2], tempty_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ int no_abort_sh[2];

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const uint32_t pad = (1024u - (smem_u32(dsmem) & 1023u)) & 1023u;
  uint8_t* smem = dsmem + pad;

  const int NT = (p.N + Cfg::OUT_COLS - 1) / Cfg::OUT_COLS;
  const int KB = p.K / BK;
  const int KB4 = (KB + 3) / 4;  // FP8 scale atoms along K (four K steps each)
  const int cluster_id = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 8);  // 4 epilogue warps in each CTA of the pair
    }
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    no_abort_sh[0] = no_abort_sh[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB0);
    prefetch_tmap(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc_pair(&tmem_base_sh, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs: barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  // the offsets and A come from the kernels before this one; a cluster past the last
  // item runs none (the same decision in both of its CTAs)
  pdl_launch_dependents();
  pdl_wait();
  const int num_pairs = __ldg(p.offsets + p.G) >> 8;
  const int total = num_pairs * NT;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer (both)
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      const int nblk = p.N / 128;
      for (int item = cluster_id; item < total && ok; item += n_clusters) {
        const PairTile t = decode_pair_item(item, NT, p, num_pairs, rank);
        const int a_row = t.m_tile * Cfg::BM;
        int b_row;
        if constexpr (Cfg::SWIGLU) b_row = t.group * p.N + t.n_tile * Cfg::OUT_COLS;   // gate or up rows
        else b_row = t.group * p.N + t.n_tile * BN + static_cast<int>(rank) * Cfg::B_HALF;
        const int wblk = t.group * nblk + (t.n_tile * Cfg::OUT_COLS) / 128;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, &abort_flag)) { ok = false; break; }
          uint8_t* sa = smem + s * Cfg::STAGE_BYTES;
          uint8_t* sb = sa + Cfg::A_BYTES;
          uint8_t* ssf = sb + Cfg::B_BYTES;
          const uint32_t bar = mapa_shared(smem_u32(&full_bar[s]), 0);
          const bool new_sf = Cfg::FP8 && (kb & 3) == 0;
          if (leader) mbar_arrive_expect_tx(&full_bar[s], 2 * (Cfg::CTA_TX - (new_sf ? 0 : Cfg::SF_BYTES)));
          tma_load_2d_pair(sa, &tmA, kb * BK, a_row, bar);
          tma_load_2d_pair(sb, (Cfg::SWIGLU && rank == 1) ? &tmB1 : &tmB0, kb * BK, b_row, bar);
          if constexpr (Cfg::FP8) {
            if (new_sf) {
              const int kb4 = kb >> 2;
              tma_load_2d_pair(ssf, &tmSfa, 0, t.m_tile * KB4 + kb4, bar);
              if constexpr (Cfg::SWIGLU) {
                tma_load_2d_pair(ssf + 512, &tmSfb0, 0, wblk * KB4 + kb4, bar);
                tma_load_2d_pair(ssf + 1024, &tmSfb1, 0, wblk * KB4 + kb4, bar);
              } else {
#pragma unroll
                for (int a = 0; a < Cfg::SFB_ATOMS; ++a)
                  tma_load_2d_pair(ssf + 512 * (1 + a), &tmSfb0, 0, (wblk + a) * KB4 + kb4, bar);
              }
            }
          }
          ++issued;
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (leader) {
        // the leader's stage barriers also count the peer's bytes: once the last stages
        // completed, no copy of either CTA is in flight
        volatile int* no_abort = &no_abort_sh[0];
        const long long back = issued < STAGES ? issued : STAGES;
        for (long long j = 0; j < back; ++j) {
          if (s == 0) { s = STAGES - 1; ph ^= 1u; } else { --s; }
          mbar_wait_bounded(&full_bar[s], ph, no_abort);
        }
        if (*no_abort) abort_flag = 1;
      }
      if (!ok) abort_flag = 1;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA (leader only)
    if (leader && lane == 0) {
      int s = 0, acc = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool ok = true;
      const uint32_t sfa_t = tmem_base + Cfg::SF_COL;
      const uint32_t sfb_t = sfa_t + 4;
      for (int item = cluster_id; item < total && ok; item += n_clusters) {
        if (!mbar_wait_bounded(&tempty_bar[acc], acc_ph ^ 1u, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * Cfg::ACC_COLS;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint32_t b0 = a0 + Cfg::A_BYTES;
          if constexpr (Cfg::FP8) {
            const uint32_t sf0 = b0 + Cfg::B_BYTES;
            if ((kb & 3) == 0) {
              tmem_cp_pair_32x128b_warpx4(sfa_t, smem_desc_rows16(sf0));
#pragma unroll
              for (int a = 0; a < Cfg::SFB_ATOMS; ++a)
                tmem_cp_pair_32x128b_warpx4(sfb_t + 4 * a, smem_desc_rows16(sf0 + 512 * (1 + a)));
            }
            const uint32_t idesc = idesc_mxf8_e4m3(256, BN, kb & 3, kb & 3);
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk)
              umma_mxf8_pair(d_tmem, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32), idesc, sfa_t,
                             sfb_t, (kb | kk) != 0);
          } else {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_f16_pair(d_tmem, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32),
                            idesc_bf16_f32(256, BN), (kb | k) != 0);
          }
          umma_commit_pair(&empty_bar[s]);  // stage free in both CTAs
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair(&tfull_bar[acc]);  // accumulator ready in both CTAs
        if (++acc == ACC_STAGES) { acc = 0; acc_ph ^= 1u; }
      }
      umma_commit_pair_local(&drain_bar);
      volatile int* no_abort = &no_abort_sh[1];
      mbar_wait_bounded(&drain_bar, 0, no_abort);
      if (!ok || *no_abort) abort_flag = 1;
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both)
    const int q = warp & 3;
    const uint32_t tempty_leader0 = mapa_shared(smem_u32(&tempty_bar[0]), 0);
    const uint32_t tempty_leader1 = mapa_shared(smem_u32(&tempty_bar[1]), 0);
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int item = cluster_id; item < total; item += n_clusters) {
      const PairTile t = decode_pair_item(item, NT, p, num_pairs, rank);
      const bool ready = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull_bar[acc], acc_ph, &abort_flag));
      if (!ready) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * Cfg::ACC_COLS;
      const int row_in_tile = q * 32 + lane;
      const long long row = static_cast<long long>(t.m_tile) * Cfg::BM + row_in_tile;
      const bool row_ok = p.counts == nullptr ||
                          row - __ldg(p.offsets + t.group) < __ldg(p.counts + t.group);
      const int col0 = t.n_tile * Cfg::OUT_COLS;
      auto release = [&]() {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc == 0 ? tempty_leader0 : tempty_leader1);
      };

      if constexpr (Cfg::EPI == EPI2_SWIGLU_BF16) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + row * p.ldo + col0;
#pragma unroll 1
        for (int c = 0; c < BN / 2; c += 32) {
          uint32_t rg[32], ru[32];
          tmem_ld_32x32b_x32(tbase + c, rg);
          tmem_ld_32x32b_x32(tbase + BN / 2 + c, ru);
          tmem_ld_wait(rg);
          reg_fence(ru);
          uint32_t packed[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            packed[i] = pack_bf16x2(silu_mul(__uint_as_float(rg[2 * i]), __uint_as_float(ru[2 * i])),
                                    silu_mul(__uint_as_float(rg[2 * i + 1]), __uint_as_float(ru[2 * i + 1])));
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
          }
        }
        release();
      } else if constexpr (Cfg::EPI == EPI2_SWIGLU_E4M3) {
        float h[128];
#pragma unroll
        for (int c = 0; c < 128; c += 32) {
          uint32_t rg[32], ru[32];
          tmem_ld_32x32b_x32(tbase + c, rg);
          tmem_ld_32x32b_x32(tbase + 128 + c, ru);
          tmem_ld_wait(rg);
          reg_fence(ru);
#pragma unroll
          for (int i = 0; i < 32; ++i) h[c + i] = silu_mul(__uint_as_float(rg[i]), __uint_as_float(ru[i]));
        }
        release();  // the accumulator is in registers: hand TMEM back before quantising
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 128; ++i) amax = fmaxf(amax, fabsf(h[i]));
        const int e = e4m3_scale_exponent(amax);
        const float inv = ldexpf(1.f, -e);
        if (row_ok) {
          uint8_t* out = static_cast<uint8_t*>(p.out) + row * p.ldo + col0;
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const float* hv = h + 16 * v;
            reinterpret_cast<uint4*>(out)[v] = make_uint4(
                e4m3x4(hv[0] * inv, hv[1] * inv, hv[2] * inv, hv[3] * inv),
                e4m3x4(hv[4] * inv, hv[5] * inv, hv[6] * inv, hv[7] * inv),
                e4m3x4(hv[8] * inv, hv[9] * inv, hv[10] * inv, hv[11] * inv),
                e4m3x4(hv[12] * inv, hv[13] * inv, hv[14] * inv, hv[15] * inv));
          }
        }
        const int kb4n = (p.N / 128 + 3) / 4;
        uint8_t* sf = p.out_sf + (static_cast<size_t>(t.m_tile) * kb4n + (t.n_tile >> 2)) * 512;
        sf[sf_atom_offset(row_in_tile) + (t.n_tile & 3)] = static_cast<uint8_t>(e + 127);
      } else if constexpr (Cfg::EPI == EPI2_F32) {
        float* out = static_cast<float*>(p.out) + row * p.ldo + col0;
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + c, r);
          tmem_ld_wait(r);
          if (row_ok && col0 + c < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
            for (int v = 0; v < 8; ++v) dst[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
          }
        }
        release();
      } else {
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
        release();
      }
      if (++acc == ACC_STAGES) { acc = 0; acc_ph ^= 1u; }
    }
  }

  __syncthreads();
  tc_fence_before();
  cluster_sync();  // both CTAs done with TMEM and with each other's barriers
  tc_fence_after();
  if (abort_flag && threadIdx.x == 0) set_status(p.status, MOE_DEV_TIMEOUT);
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace moe
