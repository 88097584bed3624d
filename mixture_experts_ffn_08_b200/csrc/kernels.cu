// Routing, dispatch and combine kernels of the MoE layer (sm_100a).
//
//   topk_kernel        warp per token: scores, selection bias, group-limited top-k,
//                      renormalised weights (routing primer "MoE 路由入门" §三, §四,
//                      §六-§十; "MoE" chapter index §0 "+bias only for selection")
//   perm_*_kernel      pairs bucketed by expert, stably, each bucket padded to the GEMM
//                      M-tile (routing primer §5.1): per-chunk histogram -> one-block scan
//                      -> stable in-chunk ranks with warp match -> row gather of x
//   combine_kernel     out_t = sum_k w_tk y_tk (+ shared), fixed k order (routing primer
//                      §5.3), vectorised, no atomics
#include <cuda_fp8.h>
#include <math_constants.h>

#include "common.cuh"
#include "internal.h"
#include "tc_gemm_fp8.cuh"  // the scale-atom layout (sf_atom_offset)

namespace moe {

constexpr unsigned kFull = 0xffffffffu;

// ================================================================== FP8 x -> bf16 (router)
// Each e4m3 value times its power-of-two scale is exactly representable in bf16.
__global__ void dequant_x_kernel(const uint8_t* __restrict__ xq, const float* __restrict__ xs,
                                 int T, int H, __nv_bfloat16* __restrict__ xb) {
  pdl_launch_dependents();
  pdl_wait();
  const long long n16 = static_cast<long long>(T) * H / 16;
  for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < n16;
       v += (long long)gridDim.x * blockDim.x) {
    const long long e0 = v * 16;
    const int t = static_cast<int>(e0 / H), h = static_cast<int>(e0 % H);
    const float s = __ldg(xs + static_cast<long long>(t) * (H / 128) + h / 128);
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(xq) + v);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>(w[i] >> (16 * half));
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
        o[2 * i + half] = pack_bf16x2(f.x * s, f.y * s);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(xb) + v * 2;
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

cudaError_t launch_dequant_x(const uint8_t* xq, const float* xs, int T, int H, void* x_bf16,
                             cudaStream_t st) {
  const long long n16 = static_cast<long long>(T) * H / 16;
  const int grid = static_cast<int>(n16 / 256 + 1 < num_sms() * 8 ? n16 / 256 + 1 : num_sms() * 8);
  trace_before(MOE_K_DEQUANT_X, st);
  const cudaError_t err = launch_k(dequant_x_kernel, grid, 256, 0, st, xq, xs, T, H,
                                   static_cast<__nv_bfloat16*>(x_bf16));
  trace_after(MOE_K_DEQUANT_X, st);
  return err != cudaSuccess ? err : cudaGetLastError();
}

// ================================================================== top-k
// (value, index) order: larger value first, equal values -> lower index first.
MOE_DEVINL bool better(float v, int i, float v2, int i2) { return v > v2 || (v == v2 && i < i2); }

MOE_DEVINL void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(kFull, v, o);
    const int i2 = __shfl_xor_sync(kFull, i, o);
    if (better(v2, i2, v, i)) { v = v2; i = i2; }
  }
}

MOE_DEVINL float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(kFull, v, o);
  return v;
}

MOE_DEVINL float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

// Lane l holds experts l, l+32, l+64, ... (EPL of them): E <= 32 * EPL, so register j
// of all lanes covers experts [32j, 32j+32).
//
// Group stage: when every group is a whole number of registers (group size a multiple
// of 32) and the group score uses at most the two best experts, all group scores come
// out of one butterfly that carries each register's top-2 across the warp, the groups'
// registers merged in parallel; every lane then ranks the groups itself.  Any other
// grouping takes the general path (one warp argmax per group and rank).
// Top-K: each lane sorts its EPL candidates (descending score, ascending expert id), so
// every one of the K rounds is a single warp argmax over the lanes' heads.
template <int EPL>
__global__ void __launch_bounds__(128) topk_kernel(
    const float* __restrict__ logits, int n_part, int T, int E, int K, int n_group, int topk_group,
    int group_topn, int score_fn, int renorm, float scale, const float* __restrict__ bias,
    int32_t* __restrict__ ids, float* __restrict__ wout) {
  pdl_launch_dependents();
  pdl_wait();
  const int token = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (token >= T) return;  // warp-uniform
  const float* z = logits + static_cast<long long>(token) * E;
  const long long part_stride = static_cast<long long>(T) * E;

  // logits: the sum of n_part partial slices, added in slice order
  float s[EPL], c[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = j * 32 + lane;
    s[j] = e < E ? __ldg(z + e) : -CUDART_INF_F;
  }
  // (U slices' loads in flight at once, then added in slice order: the same sum)
  constexpr int U = EPL <= 8 ? 4 : 1;
  int part = 1;
  for (; part + U <= n_part; part += U) {
    float a[U][EPL];
#pragma unroll
    for (int q = 0; q < U; ++q)
#pragma unroll
      for (int j = 0; j < EPL; ++j) {
        const int e = j * 32 + lane;
        a[q][j] = e < E ? __ldg(z + (part + q) * part_stride + e) : 0.f;
      }
#pragma unroll
    for (int q = 0; q < U; ++q)
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (j * 32 + lane < E) s[j] += a[q][j];
  }
  for (; part < n_part; ++part) {
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      const int e = j * 32 + lane;
      if (e < E) s[j] += __ldg(z + part * part_stride + e);
    }
  }
  if (score_fn == MOE_SCORE_SOFTMAX) {
    float m = -CUDART_INF_F;
#pragma unroll
    for (int j = 0; j < EPL; ++j) m = fmaxf(m, s[j]);
    m = warp_max(m);
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j) {
      s[j] = (j * 32 + lane < E) ? expf(s[j] - m) : 0.f;
      sum += s[j];
    }
    sum = warp_sum(sum);
#pragma unroll
    for (int j = 0; j < EPL; ++j) s[j] = s[j] / sum;
  } else {
#pragma unroll
    for (int j = 0; j < EPL; ++j) s[j] = (j * 32 + lane < E) ? 1.f / (1.f + expf(-s[j])) : 0.f;
  }
#pragma unroll
  for (int j = 0; j < EPL; ++j) {
    const int e = j * 32 + lane;
    c[j] = e < E ? s[j] + (bias ? __ldg(bias + e) : 0.f) : -CUDART_INF_F;
  }

  if (n_group > 1) {
    const int gs = E / n_group;
    uint32_t keep = 0;
    if (gs % 32 == 0 && group_topn <= 2) {
      // top-2 of every register across the warp, all registers at once
      float t1[EPL], t2[EPL];
#pragma unroll
      for (int j = 0; j < EPL; ++j) { t1[j] = c[j]; t2[j] = -CUDART_INF_F; }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
          const float b1 = __shfl_xor_sync(kFull, t1[j], o);
          const float b2 = __shfl_xor_sync(kFull, t2[j], o);
          const float hi = fmaxf(t1[j], b1);
          t2[j] = fmaxf(fminf(t1[j], b1), fmaxf(t2[j], b2));
          t1[j] = hi;
        }
      }
      // group g spans registers [g*R, (g+1)*R); merge their top-2 lists
      // here every group is at least one register, so n_group <= EPL
      const int R = gs / 32;
      float gscore[EPL];
#pragma unroll
      for (int g = 0; g < EPL; ++g) {
        float a1 = -CUDART_INF_F, a2 = -CUDART_INF_F;
#pragma unroll
        for (int j = 0; j < EPL; ++j) {
          if (j / R == g) {
            const float hi = fmaxf(a1, t1[j]);
            a2 = fmaxf(fminf(a1, t1[j]), fmaxf(a2, t2[j]));
            a1 = hi;
          }
        }
        gscore[g] = g < n_group ? (group_topn == 1 ? a1 : a1 + a2) : -CUDART_INF_F;
      }
      // rank the groups in registers (all lanes agree): best score, lower index on ties
      for (int r = 0; r < topk_group; ++r) {
        int best = -1;
        float bv = -CUDART_INF_F;
#pragma unroll
        for (int g = 0; g < EPL; ++g)
          if (g < n_group && !((keep >> g) & 1u) && (best < 0 || gscore[g] > bv)) { bv = gscore[g]; best = g; }
        keep |= 1u << best;
      }
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (j * 32 < E && !((keep >> (j / R)) & 1u)) c[j] = -CUDART_INF_F;
    } else {
      int grp[EPL];
#pragma unroll
      for (int j = 0; j < EPL; ++j) grp[j] = (j * 32 + lane) / gs;
      float my_gscore = -CUDART_INF_F;  // lane g keeps the score of group g
      for (int g = 0; g < n_group; ++g) {
        uint32_t taken = 0;
        float acc = 0.f;
        for (int r = 0; r < group_topn; ++r) {
          float bv = -CUDART_INF_F;
          int bi = 0x7fffffff;
#pragma unroll
          for (int j = 0; j < EPL; ++j) {
            const int e = j * 32 + lane;
            if (e < E && grp[j] == g && !((taken >> j) & 1u) && better(c[j], e, bv, bi)) {
              bv = c[j];
              bi = e;
            }
          }
          warp_argmax(bv, bi);
          acc += bv;
          if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        }
        if (lane == g) my_gscore = acc;
      }
      float cand = lane < n_group ? my_gscore : -CUDART_INF_F;
      for (int r = 0; r < topk_group; ++r) {
        float bv = cand;
        int bi = lane;
        warp_argmax(bv, bi);
        keep |= 1u << bi;
        if (lane == bi) cand = -CUDART_INF_F;
      }
#pragma unroll
      for (int j = 0; j < EPL; ++j)
        if (j * 32 + lane < E && !((keep >> grp[j]) & 1u)) c[j] = -CUDART_INF_F;
    }
  }

  // sort this lane's candidates: descending c, ascending expert id (insertion network)
  float sc[EPL];
  int se[EPL];
#pragma unroll
  for (int j = 0; j < EPL; ++j) { sc[j] = c[j]; se[j] = j * 32 + lane; }
#pragma unroll
  for (int a = 1; a < EPL; ++a) {
#pragma unroll
    for (int b = a; b > 0; --b) {
      if (better(sc[b], se[b], sc[b - 1], se[b - 1])) {
        const float tv = sc[b]; sc[b] = sc[b - 1]; sc[b - 1] = tv;
        const int te = se[b]; se[b] = se[b - 1]; se[b - 1] = te;
      }
    }
  }
  int my_id = -1;
  float my_w = 0.f;
  for (int k = 0; k < K; ++k) {
    float bv = sc[0];
    int bi = se[0];
    warp_argmax(bv, bi);
    const int owner = bi & 31, jj = bi >> 5;
    float sv = 0.f;
#pragma unroll
    for (int j = 0; j < EPL; ++j)
      if (j == jj) sv = s[j];
    sv = __shfl_sync(kFull, sv, owner);
    if (lane == owner) {   // pop the head
#pragma unroll
      for (int j = 0; j < EPL - 1; ++j) { sc[j] = sc[j + 1]; se[j] = se[j + 1]; }
      sc[EPL - 1] = -CUDART_INF_F;
      se[EPL - 1] = 0x7fffffff;
    }
    if (lane == k) { my_id = bi; my_w = sv; }
  }
  const float wsum = warp_sum(my_w);
  if (renorm) my_w = my_w / wsum;
  my_w *= scale;
  if (lane < K) {
    ids[static_cast<long long>(token) * K + lane] = my_id;
    wout[static_cast<long long>(token) * K + lane] = my_w;
  }
}

cudaError_t launch_topk(const float* logits, const moe_params_t& p, const float* bias,
                        int32_t* ids, float* w, cudaStream_t st, int n_part) {
  const int grid = (p.T + 3) / 4;
  if (grid == 0) return cudaSuccess;
  const int epl = (p.E + 31) / 32;
  trace_before(MOE_K_TOPK, st);
  cudaError_t err;
#define MOE_TOPK_CASE(N)                                                                             \
  err = launch_k(topk_kernel<N>, grid, 128, 0, st, logits, n_part, p.T, p.E, p.K, p.n_group,         \
                 p.topk_group, p.group_topn, static_cast<int>(p.score_fn), p.renormalize,            \
                 p.routed_scale, bias, ids, w)
  if (epl <= 1) MOE_TOPK_CASE(1);
  else if (epl <= 2) MOE_TOPK_CASE(2);
  else if (epl <= 4) MOE_TOPK_CASE(4);
  else if (epl <= 8) MOE_TOPK_CASE(8);
  else if (epl <= 16) MOE_TOPK_CASE(16);
  else MOE_TOPK_CASE(32);
#undef MOE_TOPK_CASE
  trace_after(MOE_K_TOPK, st);
  return err != cudaSuccess ? err : cudaGetLastError();
}

// ================================================================== aux-free bias
// b_e += gamma * sign(mean_load - load_e), the sign taken exactly in integers as
// sign(sum_j load_j - E * load_e).  One block.
__global__ void __launch_bounds__(1024) bias_update_kernel(const int32_t* __restrict__ counts, int E,
                                                           float gamma, float* __restrict__ bias) {
  __shared__ long long warp_sum_sh[32];
  long long local = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) local += __ldg(counts + e);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(kFull, local, o);
  if ((threadIdx.x & 31) == 0) warp_sum_sh[threadIdx.x >> 5] = local;
  __syncthreads();
  long long total = 0;
  for (int w = 0; w < (int)(blockDim.x + 31) / 32; ++w) total += warp_sum_sh[w];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const long long d = total - static_cast<long long>(E) * __ldg(counts + e);
    const float sgn = d > 0 ? 1.f : (d < 0 ? -1.f : 0.f);
    bias[e] = bias[e] + gamma * sgn;
  }
}

cudaError_t launch_bias_update(const int32_t* counts, int E, float gamma, float* bias, cudaStream_t st) {
  bias_update_kernel<<<1, 1024, 0, st>>>(counts, E, gamma, bias);
  return cudaGetLastError();
}

// ================================================================== bounded-wait self-test
// One thread waits on an mbarrier that nothing completes, with the same bounded wait
// the GEMM pipelines use, and reports the give-up as MOE_DEV_TIMEOUT.
__global__ void bounded_wait_selftest_kernel(int32_t* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns)) set_status(status, MOE_DEV_TIMEOUT);
}

cudaError_t launch_bounded_wait_selftest(int32_t* status, long long limit_ns, cudaStream_t st) {
  bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(status, static_cast<unsigned long long>(limit_ns));
  return cudaGetLastError();
}

// ================================================================== permute
// 1) per-chunk expert histogram
__global__ void __launch_bounds__(kPermChunk) perm_count_kernel(
    const int32_t* __restrict__ ids, int P, int E, int32_t* __restrict__ chunk_counts,
    int32_t* status) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ int hist[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int p = blockIdx.x * kPermChunk + threadIdx.x;
  if (p < P) {
    const int e = __ldg(ids + p);
    if (e >= 0 && e < E) atomicAdd(&hist[e], 1);
    else set_status(status, MOE_DEV_BAD_EXPERT_ID);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    chunk_counts[static_cast<long long>(blockIdx.x) * E + e] = hist[e];
}

// 2) one block: expert totals, padded exclusive scan -> offsets, and per-chunk bases
//    (chunk_counts is overwritten with the first row of each (chunk, expert) run).
//    cap > 0 (masked layout): every expert spans cap rows, counts are capped at cap.
//    Thread (part, e) handles expert e over one of 1024 / E contiguous ranges of chunks,
//    so all 1024 threads walk the chunk table, not only E of them.
__global__ void __launch_bounds__(1024) perm_scan_kernel(int32_t* __restrict__ chunk_counts,
                                                         int nchunks, int E, int block_m, int cap,
                                                         int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets,
                                                         int32_t* status) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int warp_tot[32];
  __shared__ int part_run[1024];        // [part][E]: pairs of expert e in the part's chunks, then
                                        // the pairs of e in the parts before it
  __shared__ int first_row[kMaxExperts];
  const int tid = threadIdx.x;
  const int parts = E <= 1024 ? 1024 / E : 1;
  const int per = (nchunks + parts - 1) / parts;
  const int my_part = tid / E, my_e = tid - my_part * E;
  const bool walker = my_part < parts;
  const int c0 = my_part * per, c1 = c0 + per < nchunks ? c0 + per : nchunks;
  if (walker) {
    int sum = 0;
    for (int c = c0; c < c1; ++c) sum += chunk_counts[static_cast<long long>(c) * E + my_e];
    part_run[tid] = sum;
  }
  __syncthreads();
  const int e = tid, lane = e & 31, w = e >> 5;
  int total = 0;
  if (e < E)
    for (int q = 0; q < parts; ++q) {
      const int n = part_run[q * E + e];
      part_run[q * E + e] = total;
      total += n;
    }
  const int padded = e >= E ? 0 : cap > 0 ? cap : (total + block_m - 1) / block_m * block_m;
  // inclusive scan of `padded` across the block
  int v = padded;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[w] = v;
  __syncthreads();
  if (w == 0) {
    int t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(kFull, t, o);
      if (lane >= o) t += n;
    }
    warp_tot[lane] = t;  // inclusive totals of warps 0..lane
  }
  __syncthreads();
  const int incl = v + (w > 0 ? warp_tot[w - 1] : 0);
  const int excl = incl - padded;
  if (e < E) {
    if (cap > 0 && total > cap) set_status(status, MOE_DEV_CAPACITY);
    counts[e] = cap > 0 && total > cap ? cap : total;
    offsets[e] = excl;
    first_row[e] = excl;
  }
  if (e == E - 1) offsets[E] = incl;
  __syncthreads();
  if (walker) {
    int run = first_row[my_e] + part_run[tid];
    for (int c = c0; c < c1; ++c) {
      const long long idx = static_cast<long long>(c) * E + my_e;
      const int n = chunk_counts[idx];
      chunk_counts[idx] = run;
      run += n;
    }
  }
}

// 3) stable rank inside each chunk: one warp per chunk walks its pairs in order,
//    32 at a time; lanes with the same expert are ranked by lane (warp match).
constexpr int kRankWarps = 4;
//    cap > 0 (masked layout): a pair whose row falls past its expert's cap rows gets none.
__global__ void __launch_bounds__(32 * kRankWarps) perm_rank_kernel(
    const int32_t* __restrict__ ids, int P, int E, int cap, const int32_t* __restrict__ chunk_base,
    int32_t* __restrict__ row_of_pair, int32_t* __restrict__ pair_of_row) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ int run_cnt[];  // [kRankWarps][E]
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int* my = run_cnt + w * E;
  for (int e = lane; e < E; e += 32) my[e] = 0;
  __syncwarp();
  const int chunk = blockIdx.x * kRankWarps + w;
  if (chunk * kPermChunk >= P) return;  // warp-uniform
  const int32_t* base = chunk_base + static_cast<long long>(chunk) * E;
  for (int it = 0; it < kPermChunk / 32; ++it) {
    const int p = chunk * kPermChunk + it * 32 + lane;
    const int e = p < P ? __ldg(ids + p) : -1;
    const bool ok = p < P && e >= 0 && e < E;
    const int key = ok ? e : -1 - lane;  // invalid lanes match nobody
    const unsigned peers = __match_any_sync(kFull, key);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int run = ok ? my[e] : 0;
    __syncwarp();
    if (ok) {
      const int row = __ldg(base + e) + run + rank;
      const bool kept = cap <= 0 || row < (e + 1) * cap;
      row_of_pair[p] = kept ? row : -1;
      if (kept) pair_of_row[row] = p;
      if (rank == 0) my[e] = run + __popc(peers);
    } else if (p < P) {
      row_of_pair[p] = -1;
    }
    __syncwarp();
  }
}

// 1-3 in one block, for at most kSmallPairs pairs (decode-sized batches): expert counts
// in shared memory, the padded scan, then one warp walks the pairs in order, 32 at a
// time, for the stable ranks.  Same outputs as the three kernels above.
__global__ void __launch_bounds__(1024) perm_small_kernel(
    const int32_t* __restrict__ ids, int P, int E, int block_m, int cap, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ row_of_pair, int32_t* __restrict__ pair_of_row,
    int32_t* status) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int cnt[kMaxExperts];
  __shared__ int next_row[kMaxExperts];
  __shared__ int warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  for (int e = tid; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int p = tid; p < P; p += blockDim.x) {
    const int e = __ldg(ids + p);
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    else set_status(status, MOE_DEV_BAD_EXPERT_ID);
  }
  __syncthreads();
  // padded exclusive scan over the experts (E <= blockDim.x)
  const int e = tid;
  const int total = e < E ? cnt[e] : 0;
  const int padded = e >= E ? 0 : cap > 0 ? cap : (total + block_m - 1) / block_m * block_m;
  int v = padded;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[w] = v;
  __syncthreads();
  if (w == 0) {
    int t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(kFull, t, o);
      if (lane >= o) t += n;
    }
    warp_tot[lane] = t;
  }
  __syncthreads();
  const int incl = v + (w > 0 ? warp_tot[w - 1] : 0);
  const int excl = incl - padded;
  if (e < E) {
    if (cap > 0 && total > cap) set_status(status, MOE_DEV_CAPACITY);
    counts[e] = cap > 0 && total > cap ? cap : total;
    offsets[e] = excl;
    next_row[e] = excl;
  }
  if (e == E - 1) offsets[E] = incl;
  __syncthreads();
  if (w == 0) {
    for (int base = 0; base < P; base += 32) {
      const int p = base + lane;
      const int ex = p < P ? __ldg(ids + p) : -1;
      const bool ok = p < P && ex >= 0 && ex < E;
      const int key = ok ? ex : -1 - lane;  // invalid lanes match nobody
      const unsigned peers = __match_any_sync(kFull, key);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int r0 = ok ? next_row[ex] : 0;
      __syncwarp();
      if (ok) {
        const int row = r0 + rank;
        const bool kept = cap <= 0 || row < (ex + 1) * cap;
        row_of_pair[p] = kept ? row : -1;
        if (kept) pair_of_row[row] = p;
        if (rank == 0) next_row[ex] = r0 + __popc(peers);
      } else if (p < P) {
        row_of_pair[p] = -1;
      }
      __syncwarp();
    }
  }
}

// 4) row gather: x_perm[r] = x[pair_of_row[r] / K]; pad rows -> pair -1 and, unless
//    zero_pad is false (masked layout: unused rows are left as they are), zero.
//    One warp per row; each lane keeps up to 8 16-byte loads in flight, so the copy runs
//    at HBM write speed rather than at the latency of one load per thread.
constexpr int kGatherWarps = 8;
template <bool FP8>
__global__ void __launch_bounds__(32 * kGatherWarps) perm_gather_kernel(
    const void* __restrict__ x, const float* __restrict__ x_scale, int H, int K, int E,
    const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
    int32_t* __restrict__ pair_of_row, void* __restrict__ x_perm,
    float* __restrict__ x_perm_scale, bool zero_pad) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int total = __ldg(offsets + E);
  const int row_bytes = FP8 ? H : 2 * H;
  const int nvec = row_bytes / 16;
  const int nsc = H / 128;
  const int warps = gridDim.x * kGatherWarps;
  for (int r = blockIdx.x * kGatherWarps + (threadIdx.x >> 5); r < total; r += warps) {
    int lo = 0, hi = E - 1;  // expert owning row r: smallest e with offsets[e+1] > r
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(offsets + mid + 1) > r) hi = mid; else lo = mid + 1;
    }
    const bool pad = r - __ldg(offsets + lo) >= __ldg(counts + lo);
    if (pad && lane == 0) pair_of_row[r] = -1;
    if (pad && !zero_pad) continue;
    const long long t = pad ? 0 : pair_of_row[r] / K;
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(x_perm) + static_cast<long long>(r) * row_bytes);
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(x) + t * row_bytes);
    for (int v0 = 0; v0 < nvec; v0 += 32 * 8) {
      uint4 buf[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int v = v0 + 32 * u + lane;
        buf[u] = (v < nvec && !pad) ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int v = v0 + 32 * u + lane;
        if (v < nvec) dst[v] = buf[u];
      }
    }
    if (FP8) {
      for (int j = lane; j < nsc; j += 32)
        x_perm_scale[static_cast<long long>(r) * nsc + j] = pad ? 1.0f : __ldg(x_scale + t * nsc + j);
    }
  }
}

// 4') token scatter, for the layer itself (no pad rows written, pair_of_row of pad rows not
//     needed): a warp reads a 256-vector (4 or 8 KB) piece of x[t] once and stores it to the
//     bucket rows of its K pairs, so x crosses HBM once where the row gather re-reads each
//     token K times.  Work units are (token, piece), so a decode-sized batch still spreads
//     over the SMs.
constexpr int kScatterWarps = 8;
template <bool FP8>
__global__ void __launch_bounds__(32 * kScatterWarps) perm_scatter_kernel(
    const void* __restrict__ x, const float* __restrict__ x_scale, int T, int H, int K,
    const int32_t* __restrict__ row_of_pair, void* __restrict__ x_perm, float* __restrict__ x_perm_scale,
    uint8_t* __restrict__ x_atoms) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int row_bytes = FP8 ? H : 2 * H;
  const int nvec = row_bytes / 16;
  const int nsc = H / 128;
  const int nchunk = (nvec + 255) / 256;
  const long long units = static_cast<long long>(T) * nchunk;
  const int warps = gridDim.x * kScatterWarps;
  for (long long u = blockIdx.x * kScatterWarps + (threadIdx.x >> 5); u < units; u += warps) {
    const int t = static_cast<int>(u / nchunk);
    const int chunk = static_cast<int>(u % nchunk);
    const int my_row = lane < K ? __ldg(row_of_pair + static_cast<long long>(t) * K + lane) : -1;
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(x) + static_cast<long long>(t) * row_bytes);
    {
      const int v0 = chunk * 256;
      uint4 buf[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int v = v0 + 32 * u + lane;
        buf[u] = v < nvec ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
      }
      for (int k = 0; k < K; ++k) {
        const int r = __shfl_sync(kFull, my_row, k);
        if (r < 0) continue;  // a pair left out (masked layout) or with a bad expert id
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(x_perm) + static_cast<long long>(r) * row_bytes);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int v = v0 + 32 * u + lane;
          if (v < nvec) dst[v] = buf[u];
        }
      }
    }
    if (FP8 && chunk == 0) {
      const int nsc4 = (nsc + 3) / 4;
      for (int k = 0; k < K; ++k) {
        const int r = __shfl_sync(kFull, my_row, k);
        if (r < 0) continue;
        if (x_atoms != nullptr) {
          // the block-scaled GEMM's scale atoms directly: row r's word in atom (r / 128, q)
          // holds the UE8M0 exponents of its scales 4q ... 4q + 3 (127 = 1.0 past the end)
          for (int q = lane; q < nsc4; q += 32) {
            uint32_t word = 0;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              const int j = 4 * q + b;
              const uint32_t e =
                  j < nsc ? (__float_as_uint(__ldg(x_scale + static_cast<long long>(t) * nsc + j)) >> 23) & 0xFFu
                          : 127u;
              word |= e << (8 * b);
            }
            *reinterpret_cast<uint32_t*>(x_atoms + (static_cast<long long>(r >> 7) * nsc4 + q) * 512 +
                                         sf_atom_offset(r & 127)) = word;
          }
        } else {
          for (int j = lane; j < nsc; j += 32)
            x_perm_scale[static_cast<long long>(r) * nsc + j] = __ldg(x_scale + static_cast<long long>(t) * nsc + j);
        }
      }
    }
  }
}

cudaError_t launch_permute(const moe_params_t& p, int block_m, const int32_t* ids, const void* x,
                           const float* x_scale, int32_t* counts, int32_t* offsets,
                           int32_t* row_of_pair, int32_t* pair_of_row, void* x_perm,
                           float* x_perm_scale, int32_t* chunk_counts, int32_t* status,
                           cudaStream_t st, bool fill_pad, uint8_t* x_atoms) {
  const int P = p.T * p.K;
  const int nchunks = (P + kPermChunk - 1) / kPermChunk;
  const int bm = block_m;
  cudaError_t err;
  if (P > 0 && P <= kSmallPairs) {
    trace_before(MOE_K_PERM_SCAN, st);
    err = launch_k(perm_small_kernel, 1, 1024, 0, st, ids, P, p.E, bm, p.masked_cap, counts, offsets, row_of_pair,
                   pair_of_row, status);
    trace_after(MOE_K_PERM_SCAN, st);
    if (err != cudaSuccess || (err = cudaGetLastError()) != cudaSuccess) return err;
  } else {
  if (nchunks > 0) {
    trace_before(MOE_K_PERM_COUNT, st);
    err = launch_k(perm_count_kernel, nchunks, kPermChunk, p.E * sizeof(int), st, ids, P, p.E, chunk_counts,
                   status);
    trace_after(MOE_K_PERM_COUNT, st);
    if (err != cudaSuccess || (err = cudaGetLastError()) != cudaSuccess) return err;
  }
  trace_before(MOE_K_PERM_SCAN, st);
  err = launch_k(perm_scan_kernel, 1, 1024, 0, st, chunk_counts, nchunks, p.E, bm, p.masked_cap, counts, offsets,
                 status);
  trace_after(MOE_K_PERM_SCAN, st);
  if (err != cudaSuccess || (err = cudaGetLastError()) != cudaSuccess) return err;
  if (nchunks > 0) {
    trace_before(MOE_K_PERM_RANK, st);
    const int blocks = (nchunks + kRankWarps - 1) / kRankWarps;
    err = launch_k(perm_rank_kernel, blocks, 32 * kRankWarps, kRankWarps * p.E * sizeof(int), st, ids, P, p.E,
                   p.masked_cap, chunk_counts, row_of_pair, pair_of_row);
    trace_after(MOE_K_PERM_RANK, st);
    if (err != cudaSuccess || (err = cudaGetLastError()) != cudaSuccess) return err;
  }
  }
  const bool masked = p.masked_cap > 0;
  const bool zero_pad = !masked && fill_pad;
  if (!fill_pad && p.T > 0) {
    const long long row_vecs = (act_e4m3(p) ? p.H : 2LL * p.H) / 16;
    const long long units = static_cast<long long>(p.T) * ((row_vecs + 255) / 256);
    const long long want = (units + kScatterWarps - 1) / kScatterWarps;
    const int grid = static_cast<int>(want < num_sms() * 8LL ? want : num_sms() * 8LL);
    trace_before(MOE_K_PERM_GATHER, st);
    if (act_e4m3(p))
      err = launch_k(perm_scatter_kernel<true>, grid, 32 * kScatterWarps, 0, st, x, x_scale, p.T, p.H, p.K,
                     row_of_pair, x_perm, x_perm_scale, x_atoms);
    else
      err = launch_k(perm_scatter_kernel<false>, grid, 32 * kScatterWarps, 0, st, x, x_scale, p.T, p.H, p.K,
                     row_of_pair, x_perm, x_perm_scale, static_cast<uint8_t*>(nullptr));
    trace_after(MOE_K_PERM_GATHER, st);
    return err != cudaSuccess ? err : cudaGetLastError();
  }
  const long long max_rows = masked ? static_cast<long long>(p.E) * p.masked_cap
                                    : static_cast<long long>(P) + static_cast<long long>(p.E) * (bm - 1);
  const long long blocks = (max_rows + kGatherWarps - 1) / kGatherWarps;
  const int grid = static_cast<int>(blocks < num_sms() * 8LL ? (blocks > 0 ? blocks : 1) : num_sms() * 8LL);
  trace_before(MOE_K_PERM_GATHER, st);
  if (act_e4m3(p))
    err = launch_k(perm_gather_kernel<true>, grid, 32 * kGatherWarps, 0, st, x, x_scale, p.H, p.K, p.E, counts,
                   offsets, pair_of_row, x_perm, x_perm_scale, zero_pad);
  else
    err = launch_k(perm_gather_kernel<false>, grid, 32 * kGatherWarps, 0, st, x, x_scale, p.H, p.K, p.E, counts,
                   offsets, pair_of_row, x_perm, x_perm_scale, zero_pad);
  trace_after(MOE_K_PERM_GATHER, st);
  return err != cudaSuccess ? err : cudaGetLastError();
}

// sched[e] = sum over j < e of counts[j] rounded up to 128 (one block, E <= 1024).
__global__ void __launch_bounds__(1024) masked_schedule_kernel(const int32_t* __restrict__ counts, int E,
                                                               int32_t* __restrict__ sched) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int warp_tot[32];
  const int e = threadIdx.x, lane = e & 31, w = e >> 5;
  const int padded = e < E ? (__ldg(counts + e) + 127) / 128 * 128 : 0;
  int v = padded;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[w] = v;
  __syncthreads();
  if (w == 0) {
    int t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(kFull, t, o);
      if (lane >= o) t += n;
    }
    warp_tot[lane] = t;
  }
  __syncthreads();
  const int incl = v + (w > 0 ? warp_tot[w - 1] : 0);
  if (e < E) sched[e] = incl - padded;
  if (e == E - 1) sched[E] = incl;
}

cudaError_t launch_masked_schedule(const int32_t* counts, int E, int32_t* sched, cudaStream_t st) {
  const cudaError_t err = launch_k(masked_schedule_kernel, 1, 1024, 0, st, counts, E, sched);
  return err != cudaSuccess ? err : cudaGetLastError();
}

__global__ void masked_offsets_kernel(int E, int cap, int32_t* __restrict__ offsets) {
  pdl_launch_dependents();
  pdl_wait();
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e <= E; e += gridDim.x * blockDim.x) offsets[e] = e * cap;
}

cudaError_t launch_masked_offsets(int E, int cap, int32_t* offsets, cudaStream_t st) {
  const cudaError_t err = launch_k(masked_offsets_kernel, (E + 256) / 256, 256, 0, st, E, cap, offsets);
  return err != cudaSuccess ? err : cudaGetLastError();
}

// ================================================================== combine
MOE_DEVINL void load8(const float* row, int v, float (&f)[8]) {
  const float4* src = reinterpret_cast<const float4*>(row) + 2 * v;
  const float4 a = __ldg(src), b = __ldg(src + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

MOE_DEVINL void load8(const __nv_bfloat16* row, int v, float (&f)[8]) {
  const uint4 q = __ldg(reinterpret_cast<const uint4*>(row) + v);
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

MOE_DEVINL void load8(const __half* row, int v, float (&f)[8]) {
  const uint4 q = __ldg(reinterpret_cast<const uint4*>(row) + v);
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// out[t] = sum_k w[t,k] y_perm[row_of_pair[t*K+k]] (+ y_sh[t]); YT, ST = float, bf16 or fp16.
// One block per token, with few registers (32 for the layer's fp16 and bf16 outputs), so up
// to 16 blocks share an SM and keep enough loads in flight for large batches.
template <class YT, class ST>
__global__ void __launch_bounds__(128) combine_kernel(
    const YT* __restrict__ y_perm, const int32_t* __restrict__ row_of_pair,
    const float* __restrict__ w, const ST* __restrict__ y_sh,
    __nv_bfloat16* __restrict__ out, int T, int H, int K) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int rows[kMaxTopK];
  __shared__ float wk[kMaxTopK];
  const int nvec = H / 8;  // 8 outputs (one 16-byte store) per thread step
  for (int t = blockIdx.x; t < T; t += gridDim.x) {
    __syncthreads();
    if (threadIdx.x < K) {
      rows[threadIdx.x] = __ldg(row_of_pair + static_cast<long long>(t) * K + threadIdx.x);
      wk[threadIdx.x] = __ldg(w + static_cast<long long>(t) * K + threadIdx.x);
    }
    __syncthreads();
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int k = 0; k < K; ++k) {
        const int r = rows[k];
        if (r < 0) continue;
        float f[8];
        load8(y_perm + static_cast<long long>(r) * H, v, f);
        const float wv = wk[k];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(wv, f[i], acc[i]);
      }
      if (y_sh) {
        float f[8];
        load8(y_sh + static_cast<long long>(t) * H, v, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += f[i];
      }
      reinterpret_cast<uint4*>(out + static_cast<long long>(t) * H)[v] =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                     pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    }
  }
}

// The same sum for decode-sized batches (T < 8 * SMs): a block takes one of `pieces` pieces
// of a token's H/8 output vectors, so the batch still spreads over the SMs, and each thread
// loads the rows of four pairs before it adds them, in k order (the same sum as one row at
// a time, with four loads in flight instead of one).
template <class YT, class ST>
__global__ void __launch_bounds__(128) combine_pieces_kernel(
    const YT* __restrict__ y_perm, const int32_t* __restrict__ row_of_pair,
    const float* __restrict__ w, const ST* __restrict__ y_sh,
    __nv_bfloat16* __restrict__ out, int T, int H, int K, int pieces) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ int rows[kMaxTopK];
  __shared__ float wk[kMaxTopK];
  const int nvec = H / 8;
  const int span = (nvec + pieces - 1) / pieces;
  const int units = T * pieces;
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int t = u / pieces;
    const int v0 = (u - t * pieces) * span;
    const int v1 = v0 + span < nvec ? v0 + span : nvec;
    __syncthreads();
    if (threadIdx.x < K) {
      rows[threadIdx.x] = __ldg(row_of_pair + static_cast<long long>(t) * K + threadIdx.x);
      wk[threadIdx.x] = __ldg(w + static_cast<long long>(t) * K + threadIdx.x);
    }
    __syncthreads();
    for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int k0 = 0; k0 < K; k0 += 4) {
        int r[4];
        float f[4][8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          r[j] = k0 + j < K ? rows[k0 + j] : -1;
          if (r[j] >= 0) load8(y_perm + static_cast<long long>(r[j]) * H, v, f[j]);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (r[j] < 0) continue;
          const float wv = wk[k0 + j];
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = fmaf(wv, f[j][i], acc[i]);
        }
      }
      if (y_sh) {
        float f[8];
        load8(y_sh + static_cast<long long>(t) * H, v, f);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += f[i];
      }
      reinterpret_cast<uint4*>(out + static_cast<long long>(t) * H)[v] =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                     pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
    }
  }
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ acc, long long n8, __nv_bfloat16* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait();
  for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < n8; v += (long long)gridDim.x * blockDim.x) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(acc) + 2 * v);
    const float4 b = __ldg(reinterpret_cast<const float4*>(acc) + 2 * v + 1);
    reinterpret_cast<uint4*>(out)[v] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w),
                                                  pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
  }
}

cudaError_t launch_f32_to_bf16(const float* acc, long long n, void* out, cudaStream_t st) {
  const long long n8 = n / 8;
  if (n8 == 0) return cudaSuccess;
  const long long want = (n8 + 255) / 256;
  const int grid = static_cast<int>(want < num_sms() * 8LL ? want : num_sms() * 8LL);
  trace_before(MOE_K_COMBINE, st);
  const cudaError_t err = launch_k(f32_to_bf16_kernel, grid, 256, 0, st, acc, n8, static_cast<__nv_bfloat16*>(out));
  trace_after(MOE_K_COMBINE, st);
  return err != cudaSuccess ? err : cudaGetLastError();
}

// Launches combine_kernel (pieces == 0) or combine_pieces_kernel for the output types.
template <class YT, class ST>
cudaError_t launch_combine_t(const moe_params_t& p, const void* y_perm, const int32_t* row_of_pair, const float* w,
                             const void* y_shared, void* out, cudaStream_t st, int grid, int pieces) {
  const YT* y = static_cast<const YT*>(y_perm);
  const ST* ys = static_cast<const ST*>(y_shared);
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
  if (pieces == 0) return launch_k(combine_kernel<YT, ST>, grid, 128, 0, st, y, row_of_pair, w, ys, o, p.T, p.H, p.K);
  return launch_k(combine_pieces_kernel<YT, ST>, grid, 128, 0, st, y, row_of_pair, w, ys, o, p.T, p.H, p.K, pieces);
}

cudaError_t launch_combine(const moe_params_t& p, const void* y_perm, const int32_t* row_of_pair,
                           const float* w, const void* y_shared, void* out, cudaStream_t st, bool y_f16,
                           bool ysh_f16) {
  if (p.T == 0) return cudaSuccess;
  int grid = p.T < num_sms() * 16 ? p.T : num_sms() * 16;
  int pieces = 0;
  if (p.T < num_sms() * 8) {
    // pieces per token: about eight blocks per SM, at most one piece per 128 vectors
    const int max_pieces = (p.H / 8 + 127) / 128;
    const int want = (num_sms() * 8 + p.T - 1) / p.T;
    pieces = want > max_pieces ? max_pieces : want;
    grid = p.T * pieces;
  }
  trace_before(MOE_K_COMBINE, st);
  cudaError_t err;
  if (y_f16 && ysh_f16)
    err = launch_combine_t<__half, __half>(p, y_perm, row_of_pair, w, y_shared, out, st, grid, pieces);
  else if (y_f16)
    err = launch_combine_t<__half, float>(p, y_perm, row_of_pair, w, y_shared, out, st, grid, pieces);
  else if (ysh_f16)
    err = launch_combine_t<float, __half>(p, y_perm, row_of_pair, w, y_shared, out, st, grid, pieces);
  else if (act_e4m3(p))
    err = launch_combine_t<__nv_bfloat16, float>(p, y_perm, row_of_pair, w, y_shared, out, st, grid, pieces);
  else
    err = launch_combine_t<float, float>(p, y_perm, row_of_pair, w, y_shared, out, st, grid, pieces);
  trace_after(MOE_K_COMBINE, st);
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
