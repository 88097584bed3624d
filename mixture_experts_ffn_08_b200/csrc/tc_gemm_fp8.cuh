// Block-scaled FP8 (e4m3) variant of the persistent grouped GEMM for sm_100a.
//
// Same work decomposition, warp roles and bounded waits as tc_gemm.cuh, with the MMA
// switched to tcgen05.mma.kind::mxf8f6f4.block_scale: every 32 K-elements of every row
// of A and of B carry their own UE8M0 (power-of-two) scale, applied by the tensor core.
// The layer's FP8 inputs have one power-of-two scale per 1x128 block of activations and
// per 128x128 block of weights (the FP8 workload of the layer; "SwiGLU / FP8 Cast" in the
// Mega MoE pipeline of the MoE optimisation blog §5.1), so each such scale is repeated over
// the four 32-element sub-blocks it covers and the products come out exactly as
//   sum_k (s_x[r,k/128] q_x[r,k]) (s_w[n/128,k/128] q_w[n,k]).
//
// Scales travel as 512-byte "atoms" (128 rows x one 32-bit word): row m0 + 32*m1
// (m0 < 32, m1 < 4) keeps its word at byte 16*m0 + 4*m1, and the MMA reads one byte of
// each word, chosen by the sf-id fields of the instruction descriptor.  Because the
// layer's scales cover 128 K-elements (four MX sub-blocks of 32), byte b of a word holds
// the scale of the b-th of four consecutive 128-wide K steps: one atom serves four
// pipeline stages.  Every fourth stage the producer brings the A atom and one B atom per
// 128 rows of B next to the A/B tiles (1D bulk copies on the same mbarrier); the MMA
// thread copies them to TMEM with tcgen05.cp.32x128b.warpx4 (32 lanes x 4 columns,
// replicated into the four lane quadrants) and all MMAs of K step kb select byte kb % 4.
//
// Epilogues:
//   EPI8_SWIGLU_Q  B = [128 gate rows; 128 up rows]; h = SiLU(gate) * up in fp32, then
//                  re-quantised per row and 128 columns to e4m3 with the smallest power-of-
//                  two scale that keeps |h| / scale <= 448; writes the codes and the scale
//                  atoms the down projection consumes.  One accumulator; the epilogue
//                  releases TMEM as soon as it has read it, before quantising.
//   EPI8_BF16      bf16 store (down projection), two accumulators.  The FP8 layer's
//                  2e-2 -> 6e-2 RMS bound leaves room for this rounding, and it halves
//                  the bytes of the y_perm round trip through HBM.
#pragma once

#include <cuda_fp8.h>

#include "tc_gemm.cuh"

namespace moe {

// ------------------------------------------------------------------ PTX helpers
// 1D bulk copy global -> shared (16-byte aligned, size a multiple of 16), completing on bar.
MOE_DEVINL void bulk_load(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gmem_src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Shared-memory descriptor of a K-major, unswizzled block of 16-byte rows stored back to
// back (8-row core matrices 128 bytes apart), as read by tcgen05.cp.32x128b.
MOE_DEVINL uint64_t smem_desc_rows16(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFF) >> 4);
  d |= static_cast<uint64_t>(16 >> 4) << 16;    // leading byte offset (single 16-byte column)
  d |= static_cast<uint64_t>(128 >> 4) << 32;   // stride byte offset between 8-row groups
  d |= static_cast<uint64_t>(1) << 46;          // sm_100 descriptor version
  return d;                                      // swizzle mode 0: none
}

// Copies 32 rows x 128 bits of shared memory into TMEM lanes 0-31 at `taddr` and
// replicates them into the other three 32-lane quadrants.
MOE_DEVINL void tmem_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// D[tmem] (+)= (SFA . A[smem]) * (SFB . B[smem])^T, e4m3 inputs, one UE8M0 scale per 32
// K-elements of every row, scales read from TMEM (byte a_sf_id / b_sf_id of each word).
MOE_DEVINL void umma_mxf8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                          uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Instruction descriptor, kind::mxf8f6f4 block-scaled: e4m3 A, e4m3 (b_fmt 0) or e2m1
// (b_fmt 5) B, both K-major, UE8M0 scale factors, fp32 accumulator; sf ids select the
// byte of each scale word.
constexpr uint32_t kFmtE4M3 = 0, kFmtE2M1 = 5;
__host__ __device__ constexpr uint32_t idesc_mxf8_e4m3(int M, int N, uint32_t a_sf_id,
                                                       uint32_t b_sf_id, uint32_t b_fmt = kFmtE4M3) {
  return (b_sf_id << 4)                             // B scale-factor byte
         | (kFmtE4M3 << 7) | (b_fmt << 10)          // A format e4m3, B format
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (1u << 23)                               // scale format: UE8M0
         | (static_cast<uint32_t>(M >> 4) << 24)    // M / 16
         | (a_sf_id << 29);                         // A scale-factor byte
}

// Byte offset of row m's scale word inside a 512-byte scale atom (128 rows x 4 scales of
// 32 K-elements): rows m0 + 32*m1 keep their 4 scales at 16*m0 + 4*m1.
MOE_DEVINL int sf_atom_offset(int m) { return 16 * (m & 31) + 4 * ((m >> 5) & 3); }

enum Fp8Epi { EPI8_SWIGLU_Q = 0, EPI8_BF16 = 1 };

struct Fp8Params {
  const int32_t* offsets;  // [G+1] first row of each group (multiples of 128)
  const int32_t* counts;   // [G] real rows per group (pad rows are not stored) or nullptr
  int G;
  int K;                   // reduction length, multiple of 128
  int N;                   // output columns of one group
  const uint8_t* sfa;      // A scale atoms [m_tiles][ceil(K/512)][512]
  const uint8_t* sfb0;     // B scale atoms (gate, or down weight): e4m3 [G][N/128][ceil(K/512)][512],
                           // e2m1 [G][N/128][K/128][512]
  const uint8_t* sfb1;     // up-projection scale atoms (SwiGLU only)
  void* out;               // SwiGLU: e4m3 codes [rows, ldo]; BF16: bf16 [rows, ldo]
  int64_t ldo;             // elements
  uint8_t* out_sf;         // SwiGLU: h scale atoms [m_tiles][ceil(N/512)][512]
  int32_t* status;
  int masked_cap;          // > 0: masked layout (offsets = compact schedule; rows of group g
                           // at g * masked_cap), as in GemmParams
};

// W4_: B is e2m1 (FP4) with one UE8M0 scale per 32 K: TMA unpacks 16 packed values into
// each 16-byte smem slot (8 data bytes, 8 gap bytes), so a 128-K B row fills 128 smem
// bytes exactly like e4m3; B's scale atoms then change every K step (4 scales per row).
template <int BN_, int EPI_, int STAGES_, bool W4_ = false>
struct Fp8Cfg {
  static constexpr bool W4 = W4_;
  static constexpr int BM = 128;
  static constexpr int BN = BN_;          // rows of B per tile (SwiGLU: 128 gate + 128 up)
  static constexpr int BK = 128;          // e4m3 elements (= bytes) per stage and row
  static constexpr int EPI = EPI_;
  static constexpr int STAGES = STAGES_;
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = BN * BK;                 // smem bytes of the B tile
  static constexpr int B_TX_BYTES = W4 ? B_BYTES / 2 : B_BYTES;  // bytes the TMA counts: packed e2m1
  static constexpr int SFB_ATOMS = BN / 128;
  static constexpr int SF_BYTES = 512 * (1 + SFB_ATOMS);
  static constexpr int STAGE_BYTES = (A_BYTES + B_BYTES + SF_BYTES + 1023) / 1024 * 1024;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024;
  static constexpr int OUT_COLS = EPI == EPI8_SWIGLU_Q ? BN / 2 : BN;
  // TMEM holds 512 columns: two 256-column accumulators would leave none for the scales,
  // so 256-column tiles keep one and their epilogue hands it back as soon as it is read.
  static constexpr int ACC_STAGES = BN == 256 ? 1 : 2;
  static constexpr int ACC_COLS = BN;
  static constexpr int SF_COL = ACC_STAGES * ACC_COLS;      // A scales; B scales at +4
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 192;
  static_assert(BN % 128 == 0 && BN <= 256, "B tile rows in whole 128-row scale atoms");
  static_assert(SF_COL + 4 + 4 * SFB_ATOMS <= TMEM_COLS, "TMEM columns");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(EPI != EPI8_SWIGLU_Q || BN == 256, "SwiGLU tile = 128 gate + 128 up rows");
};

// Smallest e with amax <= 448 * 2^e (e = 0 when amax == 0), exactly in fp32.  A row with
// no finite maximum (pad rows of the masked layout hold whatever the workspace held) gets
// the largest exponent at once: the search below would otherwise walk down from ilogb(inf).
MOE_DEVINL int e4m3_scale_exponent(float amax) {
  if (!(amax > 0.f)) return 0;
  if (isinf(amax)) return 127;
  int e = ilogbf(amax) - 8;
  while (amax > ldexpf(448.f, e)) ++e;
  while (e > -126 && amax <= ldexpf(448.f, e - 1)) --e;
  return e < -126 ? -126 : (e > 127 ? 127 : e);
}

MOE_DEVINL uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    tc_gemm_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmB1, const Fp8Params p) {
  constexpr int BM = Cfg::BM, BN = Cfg::BN, BK = Cfg::BK, STAGES = Cfg::STAGES;
  constexpr int ACC_STAGES = Cfg::ACC_STAGES;

  extern __shared__ uint8_t dsmem[];
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ uint64_t tfull_bar[2], tempty_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ int no_abort_sh[2];

  const int warp = warp_id(), lane = lane_id();
  const uint32_t pad = (1024u - (smem_u32(dsmem) & 1023u)) & 1023u;
  uint8_t* smem = dsmem + pad;

  const int NT = (p.N + Cfg::OUT_COLS - 1) / Cfg::OUT_COLS;
  const int KB = p.K / BK;
  const int KB4 = (KB + 3) / 4;  // scale atoms along K (four K steps each)

  // the item decoder of the bf16 kernel works on these fields only
  GemmParams gp{};
  gp.offsets = p.offsets;
  gp.G = p.G;
  gp.masked_cap = p.masked_cap;

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
    no_abort_sh[0] = no_abort_sh[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB0);
    if (Cfg::EPI == EPI8_SWIGLU_Q) prefetch_tmap(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;
  // the offsets, A and its scale atoms come from the kernels before this one
  pdl_launch_dependents();
  pdl_wait();
  const int num_m_tiles = __ldg(p.offsets + p.G) >> 7;
  const int total = num_m_tiles * NT;  // CTAs past it run no item

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      const int nblk = p.N / 128;  // 128-row weight blocks per group
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const TileCoord t = decode_item(item, NT, gp, num_m_tiles, BN);
        const int a_row = t.row0;
        const int b_row = t.group * p.N + t.n_tile * Cfg::OUT_COLS;
        const int wblk = t.group * nblk + (t.n_tile * Cfg::OUT_COLS) / 128;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, &abort_flag)) { ok = false; break; }
          uint8_t* sa = smem + s * Cfg::STAGE_BYTES;
          uint8_t* sb = sa + Cfg::A_BYTES;
          uint8_t* ssf = sb + Cfg::B_BYTES;
          const bool new_sf = (kb & 3) == 0;            // A atoms: one per four K steps
          const bool new_sfb = Cfg::W4 || new_sf;        // B atoms: every step for e2m1
          mbar_arrive_expect_tx(&full_bar[s], Cfg::A_BYTES + Cfg::B_TX_BYTES + (new_sf ? 512 : 0) +
                                                  (new_sfb ? 512 * Cfg::SFB_ATOMS : 0));
          tma_load_2d(sa, &tmA, kb * BK, a_row, &full_bar[s]);
          if (Cfg::EPI == EPI8_SWIGLU_Q) {
            tma_load_2d(sb, &tmB0, kb * BK, b_row, &full_bar[s]);
            tma_load_2d(sb + 128 * BK, &tmB1, kb * BK, b_row, &full_bar[s]);
          } else {
            tma_load_2d(sb, &tmB0, kb * BK, b_row, &full_bar[s]);
          }
          if (new_sf)
            bulk_load(ssf, p.sfa + (static_cast<size_t>(t.row0 / BM) * KB4 + (kb >> 2)) * 512, 512, &full_bar[s]);
          if (new_sfb) {
            // weight atoms [128-row block][K step (e2m1) or four K steps (e4m3)][512 B]
            const int steps = Cfg::W4 ? KB : KB4;
            const size_t wsf = (static_cast<size_t>(wblk) * steps + (Cfg::W4 ? kb : kb >> 2)) * 512;
            if (Cfg::EPI == EPI8_SWIGLU_Q) {
              bulk_load(ssf + 512, p.sfb0 + wsf, 512, &full_bar[s]);
              bulk_load(ssf + 1024, p.sfb1 + wsf, 512, &full_bar[s]);
            } else {
#pragma unroll
              for (int a = 0; a < Cfg::SFB_ATOMS; ++a)
                bulk_load(ssf + 512 * (1 + a), p.sfb0 + wsf + static_cast<size_t>(a) * steps * 512, 512,
                          &full_bar[s]);
            }
          }
          ++issued;
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      volatile int* no_abort = &no_abort_sh[0];
      const long long back = issued < STAGES ? issued : STAGES;
      for (long long j = 0; j < back; ++j) {
        if (s == 0) { s = STAGES - 1; ph ^= 1u; } else { --s; }
        mbar_wait_bounded(&full_bar[s], ph, no_abort);
      }
      if (!ok || *no_abort) abort_flag = 1;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0, acc = 0;
      uint32_t ph = 0, acc_ph = 0;
      bool ok = true;
      const uint32_t sfa_t = tmem_base + Cfg::SF_COL;
      const uint32_t sfb_t = sfa_t + 4;
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
        if (!mbar_wait_bounded(&tempty_bar[acc], acc_ph ^ 1u, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * Cfg::ACC_COLS;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint32_t b0 = a0 + Cfg::A_BYTES;
          const uint32_t sf0 = b0 + Cfg::B_BYTES;
          // new scale atoms into TMEM (tcgen05.cp and tcgen05.mma of one thread run in
          // issue order, so the MMAs of earlier steps still read the old columns)
          if ((kb & 3) == 0) tmem_cp_32x128b_warpx4(sfa_t, smem_desc_rows16(sf0));
          if (Cfg::W4 || (kb & 3) == 0) {
#pragma unroll
            for (int a = 0; a < Cfg::SFB_ATOMS; ++a)
              tmem_cp_32x128b_warpx4(sfb_t + 4 * a, smem_desc_rows16(sf0 + 512 * (1 + a)));
          }
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // A: byte kb%4 (one scale per 128 K); B: byte kk of this step's atom (e2m1,
            // one scale per 32 K) or byte kb%4 (e4m3)
            const uint32_t idesc = Cfg::W4 ? idesc_mxf8_e4m3(BM, BN, kb & 3, kk, kFmtE2M1)
                                           : idesc_mxf8_e4m3(BM, BN, kb & 3, kb & 3);
            umma_mxf8(d_tmem, smem_desc_sw128(a0 + kk * 32), smem_desc_sw128(b0 + kk * 32), idesc, sfa_t, sfb_t,
                      (kb | kk) != 0);
          }
          umma_commit(&empty_bar[s]);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);
        if (++acc == ACC_STAGES) { acc = 0; acc_ph ^= 1u; }
      }
      umma_commit(&drain_bar);
      volatile int* no_abort = &no_abort_sh[1];
      mbar_wait_bounded(&drain_bar, 0, no_abort);
      if (!ok || *no_abort) abort_flag = 1;
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      const TileCoord t = decode_item(item, NT, gp, num_m_tiles, BN);
      const bool ready = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull_bar[acc], acc_ph, &abort_flag));
      if (!ready) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * Cfg::ACC_COLS;
      const int row_in_tile = q * 32 + lane;
      const long long row = static_cast<long long>(t.row0) + row_in_tile;
      const bool row_ok = p.counts == nullptr || t.local0 + row_in_tile < __ldg(p.counts + t.group);
      const int col0 = t.n_tile * Cfg::OUT_COLS;

      if constexpr (Cfg::EPI == EPI8_SWIGLU_Q) {
        // h = SiLU(g) * u in fp32 (h is rounded to e4m3 next, and an intermediate rounding
        // of g, u or h would move some values across e4m3 rounding boundaries).  The
        // first 64 columns are computed while the accumulator is held; the last 64 are
        // read raw into registers, the accumulator goes back to the MMA warp, and their
        // SwiGLU runs after the release.
        float h[128];
#pragma unroll
        for (int c = 0; c < 64; c += 32) {
          uint32_t rg[32], ru[32];
          tmem_ld_32x32b_x32(tbase + c, rg);
          tmem_ld_32x32b_x32(tbase + 128 + c, ru);
          tmem_ld_wait(rg);
          reg_fence(ru);
#pragma unroll
          for (int i = 0; i < 32; ++i) h[c + i] = silu_mul(__uint_as_float(rg[i]), __uint_as_float(ru[i]));
        }
        {
          uint32_t rg0[32], ru0[32], rg1[32], ru1[32];
          tmem_ld_32x32b_x32(tbase + 64, rg0);
          tmem_ld_32x32b_x32(tbase + 128 + 64, ru0);
          tmem_ld_32x32b_x32(tbase + 96, rg1);
          tmem_ld_32x32b_x32(tbase + 128 + 96, ru1);
          tmem_ld_wait(rg0);
          reg_fence(ru0);
          reg_fence(rg1);
          reg_fence(ru1);
          tc_fence_before();
          mbar_arrive(&tempty_bar[acc]);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            h[64 + i] = silu_mul(__uint_as_float(rg0[i]), __uint_as_float(ru0[i]));
            h[96 + i] = silu_mul(__uint_as_float(rg1[i]), __uint_as_float(ru1[i]));
          }
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 128; ++i) amax = fmaxf(amax, fabsf(h[i]));
        const int e = e4m3_scale_exponent(amax);
        const float inv = ldexpf(1.f, -e);
        if (row_ok) {
          uint8_t* out = static_cast<uint8_t*>(p.out) + row * p.ldo + col0;
          const bool v8 = ((reinterpret_cast<uintptr_t>(p.out) | static_cast<uintptr_t>(p.ldo)) & 31) == 0;
#pragma unroll
          for (int v = 0; v < 4; ++v) {  // 32 codes per 32-byte segment
            uint32_t w[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float* hv = h + 32 * v + 4 * j;
              w[j] = e4m3x4(hv[0] * inv, hv[1] * inv, hv[2] * inv, hv[3] * inv);
            }
            if (v8) {
              st_global_v8(out + 32 * v, w);
            } else {
              reinterpret_cast<uint4*>(out + 32 * v)[0] = make_uint4(w[0], w[1], w[2], w[3]);
              reinterpret_cast<uint4*>(out + 32 * v)[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
          }
        }
        // byte (n_tile % 4) of this row's word in atom (row0 / 128, n_tile / 4) of the down GEMM
        const int kb4n = (p.N / 128 + 3) / 4;
        uint8_t* sf = p.out_sf + (static_cast<size_t>(t.row0 / BM) * kb4n + (t.n_tile >> 2)) * 512;
        sf[sf_atom_offset(row_in_tile) + (t.n_tile & 3)] = static_cast<uint8_t>(e + 127);
      } else if constexpr (ACC_STAGES == 1) {
        // one accumulator: read it all as bf16 pairs, release it, then store
        uint32_t pk[BN / 2];
#pragma unroll
        for (int c = 0; c < BN; c += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tbase + c, r);
          tmem_ld_wait(r);
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[c / 2 + i] = pack_bf16x2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
        }
        tc_fence_before();
        mbar_arrive(&tempty_bar[acc]);
        if (row_ok) {
          __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + row * p.ldo + col0;
          const bool v8 = ((reinterpret_cast<uintptr_t>(p.out) | (static_cast<uintptr_t>(p.ldo) * 2)) & 31) == 0;
#pragma unroll
          for (int c = 0; c < BN; c += 32) {
            if (col0 + c < p.N) {
              if (v8) {
                st_global_v8(out + c, pk + c / 2);
                st_global_v8(out + c + 16, pk + c / 2 + 8);
              } else {
                uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
                for (int v = 0; v < 4; ++v)
                  dst[v] = make_uint4(pk[c / 2 + 4 * v], pk[c / 2 + 4 * v + 1], pk[c / 2 + 4 * v + 2],
                                      pk[c / 2 + 4 * v + 3]);
              }
            }
          }
        }
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
        tc_fence_before();
        mbar_arrive(&tempty_bar[acc]);
      }
      if (++acc == ACC_STAGES) { acc = 0; acc_ph ^= 1u; }
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
