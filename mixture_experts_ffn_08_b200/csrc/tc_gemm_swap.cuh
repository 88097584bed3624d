// Swap-A/B gate/up + SwiGLU for e2m1 (FP4) expert weights when each expert receives only a
// few tokens (decode).
//
// With 128-row token tiles, an expert holding four tokens leaves 124 of the 128 rows of
// its M-tile as padding, and the block-scaled MMA spends its time on those rows while the
// weight stream waits.  Here the two operands trade places, as in the "Swap A/B" tiles of
// the DeepGEMM Mega MoE design ("DeepGEMM质变…" §5): 128 weight rows (output features) are
// the M operand, and the expert's tokens, in tiles of 32, are the N operand:
//
//   D_gate[f, t] = sum_k (s_w q_wgate)[g*I + f0 + f, k] (s_x q_x)[r0 + t, k]    (D_up alike)
//
// so each weight tile costs the MMA work of 32 token columns instead of 128 token rows.
// The result is the same h (and h scale atoms) the M-tile kernel writes, so the down
// projection is unchanged.
//
// Work items are (expert g, token tile j, feature tile n), laid out expert by expert from
// a schedule tsched[g] = sum_{e<g} ceil(counts[e]/32); inside an expert the token tiles of a
// feature tile are adjacent, so CTAs running side by side share each weight tile in L2.
// Token tile j of expert g covers bucket rows offsets[g] + 32j .. +31 (inside the bucket,
// whose size is a multiple of 128 and at least counts[g]).
//
// Pipeline (one CTA per SM, 192 threads): warp 0 issues the TMA loads of the gate and up
// weight tiles (128 rows x 128 K, e2m1 unpacked to one byte per value in shared memory),
// the 32-row token tile and the scale atoms; warp 1 owns TMEM and issues two MMAs (gate,
// up) per 32 K; warps 2-5 run the epilogue.  Scales: the weights' per-32-K atoms are the
// A scales (byte kk of each word for MMA kk of a K step); the tokens' 1x128 scales come in
// padded atoms made by swap_token_atoms_kernel, one per token tile and four K steps, whose
// row t holds token t's four step scales in all four words, so the B scales of every MMA
// are byte kb % 4 of the word of lane t.
//
// Epilogue: h = SiLU(gate) * up in fp32 for 32 tokens x 128 features (warp q holds
// features 32q..32q+31, one per lane); the e4m3 scale of a token's 128 features needs the
// amax over all four warps, exchanged through shared memory behind a bounded mbarrier;
// then the codes are written (one byte per lane and token) and warp 0 of the four writes
// each token's scale byte into the down projection's atoms.
//
// Every wait is bounded; on timeout the CTA sets MOE_DEV_TIMEOUT, drains what it issued,
// frees TMEM and exits.
#pragma once

#include "tc_gemm_fp8.cuh"

namespace moe {

struct SwapCfg {
  static constexpr int BM = 128;                         // weight rows (features) per tile
  static constexpr int BT = 32;                          // token rows per tile: the MMA N
  static constexpr int BK = 128;                         // K elements per stage
  static constexpr int STAGES = 5;
  static constexpr int W_BYTES = BM * BK;                // smem bytes of one unpacked weight tile
  static constexpr int W_TX = W_BYTES / 2;               // packed e2m1 bytes the TMA counts
  static constexpr int X_BYTES = BT * BK;                // e4m3 token tile
  static constexpr int STAGE_BYTES = 2 * W_BYTES + X_BYTES;  // gate | up | tokens
  static constexpr int SF_STAGE = 3 * 512;               // gate atom | up atom | token atom
  static constexpr int SMEM_BYTES = STAGES * (STAGE_BYTES + SF_STAGE) + 1024;
  static constexpr int ACC_STAGES = 2;
  static constexpr int ACC_COLS = 2 * BT;                // gate columns | up columns
  static constexpr int SF_COL = ACC_STAGES * ACC_COLS;   // gate atom; up atom +4; token atom +8
  static constexpr int TMEM_COLS = 256;
  static constexpr int THREADS = 192;
  static_assert(STAGE_BYTES % 1024 == 0, "128-byte-swizzled tiles start on 1024-byte boundaries");
  static_assert(SF_COL + 12 <= TMEM_COLS, "TMEM columns");
  static_assert(SMEM_BYTES + 2048 <= 227 * 1024, "shared memory (dynamic + static)");
};

struct SwapParams {
  const int32_t* offsets;   // [G+1] first bucket row of each expert (contiguous or e*cap)
  const int32_t* counts;    // [G] tokens of each expert
  const int32_t* tsched;    // [G+1] token-tile schedule, tsched[G] = token tiles in all
  int G;
  int K;                    // H, multiple of 128
  int N;                    // I: output features of one expert, multiple of 128
  const uint8_t* sfw0;      // gate weight atoms [G][N/128][K/128][512] (per-32-K scales)
  const uint8_t* sfw1;      // up weight atoms, same layout
  const uint8_t* sft;       // token atoms [token tiles][ceil(K/512)][512]
  uint8_t* out;             // h e4m3 codes [rows, N]
  uint8_t* out_sf;          // h scale atoms [rows/128][ceil(N/512)][512]
  int32_t* status;
};

// Instruction descriptor, kind::mxf8f6f4 block-scaled: e2m1 A (weights), e4m3 B (tokens),
// both K-major, UE8M0 scales, fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_mx_e2m1_e4m3(int M, int N, uint32_t a_sf_id, uint32_t b_sf_id) {
  return (b_sf_id << 4)                             // B scale-factor byte
         | (kFmtE2M1 << 7) | (kFmtE4M3 << 10)       // A e2m1, B e4m3
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (1u << 23)                               // scale format: UE8M0
         | (static_cast<uint32_t>(M >> 4) << 24)    // M / 16
         | (a_sf_id << 29);                         // A scale-factor byte
}

struct SwapCoord {
  int group, j, n, v;       // expert, token tile inside it, feature tile, token tile overall
};

// Item -> (expert, token tile, feature tile).  Items of expert g occupy
// [tsched[g]*NT, tsched[g+1]*NT); inside, feature tiles are outer and token tiles inner.
MOE_DEVINL SwapCoord decode_swap_item(int item, int NT, const SwapParams& p) {
  const int v = item / NT;  // a token tile of the same expert
  int lo = 0, hi = p.G - 1;  // smallest g with tsched[g+1] > v
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(p.tsched + mid + 1) > v) hi = mid; else lo = mid + 1;
  }
  const int ts0 = __ldg(p.tsched + lo);
  const int cnt = __ldg(p.tsched + lo + 1) - ts0;
  const int local = item - ts0 * NT;
  SwapCoord c;
  c.group = lo;
  c.n = local / cnt;
  c.j = local % cnt;
  c.v = ts0 + c.j;
  return c;
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    tc_gemm_swap_kernel(const __grid_constant__ CUtensorMap tmWg, const __grid_constant__ CUtensorMap tmWu,
                        const __grid_constant__ CUtensorMap tmX, const SwapParams p) {
  constexpr int BM = Cfg::BM, BT = Cfg::BT, BK = Cfg::BK, STAGES = Cfg::STAGES;
  constexpr int ACC_STAGES = Cfg::ACC_STAGES;

  extern __shared__ uint8_t dsmem[];
  __shared__ uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ uint64_t tfull_bar[ACC_STAGES], tempty_bar[ACC_STAGES], amax_bar[ACC_STAGES], drain_bar;
  __shared__ uint32_t tmem_base_sh;
  __shared__ volatile int abort_flag;
  __shared__ int no_abort_sh[2];
  __shared__ float amax_sh[ACC_STAGES][4][32];

  const int warp = warp_id(), lane = lane_id();
  const uint32_t pad = (1024u - (smem_u32(dsmem) & 1023u)) & 1023u;
  uint8_t* smem = dsmem + pad;
  uint8_t* sf_ring = smem + STAGES * Cfg::STAGE_BYTES;

  const int NT = p.N / BM;
  const int total = __ldg(p.tsched + p.G) * NT;
  const int KB = p.K / BK;
  const int KB4 = (KB + 3) / 4;
  if ((int)blockIdx.x >= total) return;  // uniform across the CTA: nothing allocated yet

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < ACC_STAGES; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 128);
      mbar_init(&amax_bar[a], 128);
    }
    mbar_init(&drain_bar, 1);
    abort_flag = 0;
    no_abort_sh[0] = no_abort_sh[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmWg);
    prefetch_tmap(&tmWu);
    prefetch_tmap(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(&tmem_base_sh, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_sh;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
        const SwapCoord c = decode_swap_item(item, NT, p);
        const int w_row = c.group * p.N + c.n * BM;
        const int x_row = __ldg(p.offsets + c.group) + c.j * BT;
        const size_t wblk = static_cast<size_t>(c.group) * NT + c.n;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[s], ph ^ 1u, &abort_flag)) { ok = false; break; }
          uint8_t* sg = smem + s * Cfg::STAGE_BYTES;
          uint8_t* su = sg + Cfg::W_BYTES;
          uint8_t* sx = su + Cfg::W_BYTES;
          uint8_t* ssf = sf_ring + s * Cfg::SF_STAGE;
          const bool new_tok = (kb & 3) == 0;  // token atoms: one per four K steps
          mbar_arrive_expect_tx(&full_bar[s], 2 * Cfg::W_TX + Cfg::X_BYTES + 1024 + (new_tok ? 512 : 0));
          tma_load_2d(sg, &tmWg, kb * BK, w_row, &full_bar[s]);
          tma_load_2d(su, &tmWu, kb * BK, w_row, &full_bar[s]);
          tma_load_2d(sx, &tmX, kb * BK, x_row, &full_bar[s]);
          const size_t wsf = (wblk * KB + kb) * 512;
          bulk_load(ssf, p.sfw0 + wsf, 512, &full_bar[s]);
          bulk_load(ssf + 512, p.sfw1 + wsf, 512, &full_bar[s]);
          if (new_tok)
            bulk_load(ssf + 1024, p.sft + (static_cast<size_t>(c.v) * KB4 + (kb >> 2)) * 512, 512, &full_bar[s]);
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
      const uint32_t sfg_t = tmem_base + Cfg::SF_COL;
      const uint32_t sfu_t = sfg_t + 4;
      const uint32_t sft_t = sfg_t + 8;
      for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
        if (!mbar_wait_bounded(&tempty_bar[acc], acc_ph ^ 1u, &abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_gate = tmem_base + acc * Cfg::ACC_COLS;
        const uint32_t d_up = d_gate + BT;
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait_bounded(&full_bar[s], ph, &abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t g0 = smem_u32(smem + s * Cfg::STAGE_BYTES);
          const uint32_t u0 = g0 + Cfg::W_BYTES;
          const uint32_t x0 = u0 + Cfg::W_BYTES;
          const uint32_t sf0 = smem_u32(sf_ring + s * Cfg::SF_STAGE);
          // scale atoms into TMEM (issued in order with the MMAs of this thread, so the MMAs
          // of earlier steps still read the previous columns)
          if ((kb & 3) == 0) tmem_cp_32x128b_warpx4(sft_t, smem_desc_rows16(sf0 + 1024));
          tmem_cp_32x128b_warpx4(sfg_t, smem_desc_rows16(sf0));
          tmem_cp_32x128b_warpx4(sfu_t, smem_desc_rows16(sf0 + 512));
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // A (weights): byte kk of the step's atom; B (tokens): byte kb % 4
            const uint32_t idesc = idesc_mx_e2m1_e4m3(BM, BT, kk, kb & 3);
            const uint64_t xd = smem_desc_sw128(x0 + kk * 32);
            const uint32_t accum = (kb | kk) != 0;
            umma_mxf8(d_gate, smem_desc_sw128(g0 + kk * 32), xd, idesc, sfg_t, sft_t, accum);
            umma_mxf8(d_up, smem_desc_sw128(u0 + kk * 32), xd, idesc, sfu_t, sft_t, accum);
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
    const int q = warp & 3;  // TMEM lanes 32q..32q+31: features 32q + lane of the tile
    const int nk4 = (p.N / 128 + 3) / 4;
    int acc = 0;
    uint32_t acc_ph = 0;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      const SwapCoord c = decode_swap_item(item, NT, p);
      const bool ready = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull_bar[acc], acc_ph, &abort_flag));
      if (!ready) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * Cfg::ACC_COLS;
      uint32_t rg[32], ru[32];
      tmem_ld_32x32b_x32(tbase, rg);
      tmem_ld_32x32b_x32(tbase + BT, ru);
      tmem_ld_wait(rg);
      reg_fence(ru);
      tc_fence_before();
      mbar_arrive(&tempty_bar[acc]);

      // h for this lane's feature and the tile's 32 tokens, fp32 (an intermediate rounding
      // would move values across e4m3 rounding boundaries)
      float h[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) h[t] = silu_mul(__uint_as_float(rg[t]), __uint_as_float(ru[t]));
      // per token: max over this warp's 32 features, left in lane t
      float mine = 0.f;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        float m = fabsf(h[t]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == t) mine = m;
      }
      amax_sh[acc][q][lane] = mine;
      mbar_arrive(&amax_bar[acc]);
      const bool agreed = __all_sync(0xffffffffu, mbar_wait_bounded(&amax_bar[acc], acc_ph, &abort_flag));
      if (!agreed) break;
      // lane t: token t's amax over the tile's 128 features, and its scale exponent
      const float amax = fmaxf(fmaxf(amax_sh[acc][0][lane], amax_sh[acc][1][lane]),
                               fmaxf(amax_sh[acc][2][lane], amax_sh[acc][3][lane]));
      const int e = e4m3_scale_exponent(amax);

      const long long r0 = static_cast<long long>(__ldg(p.offsets + c.group)) + c.j * BT;
      const int valid = __ldg(p.counts + c.group) - c.j * BT;  // real tokens in this tile
      uint8_t* out = p.out + r0 * p.N + c.n * BM + q * 32 + lane;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const int et = __shfl_sync(0xffffffffu, e, t);
        if (t < valid) {
          const float v = h[t] * ldexpf(1.f, -et);
          out[static_cast<long long>(t) * p.N] =
              static_cast<uint8_t>(__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3));
        }
      }
      if (q == 0) {
        // byte (n % 4) of token row r's word in atom (r / 128, n / 4) of the down GEMM
        const long long r = r0 + lane;
        uint8_t* sf = p.out_sf + (static_cast<size_t>(r >> 7) * nk4 + (c.n >> 2)) * 512;
        sf[sf_atom_offset(static_cast<int>(r & 127)) + (c.n & 3)] = static_cast<uint8_t>(e + 127);
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
