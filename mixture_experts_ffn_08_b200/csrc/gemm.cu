// Host side of the tcgen05 GEMMs: TMA tensor maps and the launch configurations used
// for the router logits, the gate/up projection with fused SwiGLU and the down
// projection.
#include <cudaTypedefs.h>

#include "internal.h"
#include "tc_gemm.cuh"
#include "tc_gemm_dual.cuh"

namespace moe {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// Row-major bf16 matrix [rows, cols], box of 64 columns (128 bytes) x box_rows rows,
// 128-byte swizzle; out-of-range rows read as zero.
bool make_tmap_bf16(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols,
                    uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <class Cfg>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                   const GemmParams& gp, long long max_items, int kid, cudaStream_t st) {
  auto kern = tc_gemm_kernel<Cfg>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  const long long sms = num_sms();
  const int grid = static_cast<int>(max_items < sms ? (max_items > 0 ? max_items : 1) : sms);
  trace_before(kid, st);
  err = launch_k(kern, grid, Cfg::THREADS, Cfg::SMEM_BYTES, st, a, b0, b1, gp);
  trace_after(kid, st);
  return err != cudaSuccess ? err : cudaGetLastError();
}

long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }

}  // namespace

cudaError_t gemm_router(const void* x, const void* w_r, int T, int H, int E, float* logits,
                        int32_t* status, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  const int bn = E >= 256 ? 256 : ((E + 15) / 16) * 16;
  CUtensorMap ta, tb;
  if (!make_tmap_bf16(&ta, x, T, H, 128) || !make_tmap_bf16(&tb, w_r, E, H, bn))
    return cudaErrorInvalidValue;
  GemmParams gp{};
  gp.offsets = nullptr;
  gp.counts = nullptr;
  gp.G = 1;
  gp.dense_rows = T;
  gp.K = H;
  gp.N = E;
  gp.b_rows_per_group = E;
  gp.out = logits;
  gp.ldo = E;
  gp.status = status;
  gp.k_splits = router_k_splits(T, H, E);
  gp.split_stride = static_cast<long long>(T) * E;
  const long long items = ceil_div(T, 128) * ceil_div(E, bn) * gp.k_splits;
#define MOE_ROUTER_CASE(BN, ST) \
  return launch<GemmCfg<BN, EPI_F32, ST>>(ta, tb, tb, gp, items, MOE_K_ROUTER_GEMM, st)
  switch (bn) {
    case 16: MOE_ROUTER_CASE(16, 8);
    case 32: MOE_ROUTER_CASE(32, 8);
    case 48: MOE_ROUTER_CASE(48, 8);
    case 64: MOE_ROUTER_CASE(64, 8);
    case 80: MOE_ROUTER_CASE(80, 6);
    case 96: MOE_ROUTER_CASE(96, 6);
    case 112: MOE_ROUTER_CASE(112, 6);
    case 128: MOE_ROUTER_CASE(128, 6);
    case 144: MOE_ROUTER_CASE(144, 5);
    case 160: MOE_ROUTER_CASE(160, 5);
    case 176: MOE_ROUTER_CASE(176, 5);
    case 192: MOE_ROUTER_CASE(192, 5);
    case 208: MOE_ROUTER_CASE(208, 4);
    case 224: MOE_ROUTER_CASE(224, 4);
    case 240: MOE_ROUTER_CASE(240, 4);
    default: MOE_ROUTER_CASE(256, 4);
  }
#undef MOE_ROUTER_CASE
}

cudaError_t gemm_gateup_swiglu(const void* A, int64_t a_rows, const int32_t* offsets,
                               const int32_t* counts, int G, int dense_rows, const void* w_gate,
                               const void* w_up, int N, int K, void* h, int32_t* status, int kid,
                               cudaStream_t st, int masked_cap) {
  using Cfg = GemmCfg<256, EPI_SWIGLU, 4>;
  CUtensorMap ta, tg, tu;
  if (!make_tmap_bf16(&ta, A, a_rows, K, 128) ||
      !make_tmap_bf16(&tg, w_gate, static_cast<uint64_t>(G) * N, K, 128) ||
      !make_tmap_bf16(&tu, w_up, static_cast<uint64_t>(G) * N, K, 128))
    return cudaErrorInvalidValue;
  GemmParams gp{};
  gp.offsets = offsets;
  gp.counts = counts;
  gp.G = G;
  gp.dense_rows = dense_rows;
  gp.K = K;
  gp.N = N;
  gp.b_rows_per_group = N;
  gp.out = h;
  gp.ldo = N;
  gp.status = status;
  gp.masked_cap = masked_cap;
  gp.half_tiles = 1;
  const long long items = ceil_div(a_rows, 128) * ceil_div(N, Cfg::OUT_COLS);
  return launch<Cfg>(ta, tg, tu, gp, items, kid, st);
}

cudaError_t gemm_gateup_swiglu_dual(const void* A, int64_t a_rows, const int32_t* offsets, const int32_t* counts,
                                    int G, const void* w_gate, const void* w_up, int N, int K, void* h,
                                    int32_t* counter, int32_t* status, cudaStream_t st, int masked_cap, int kid,
                                    const DualExtra* extra) {
  if (G > kDualMaxGroups || N % 128 != 0 || K % 64 != 0) return cudaErrorInvalidValue;
  const bool has_x = extra != nullptr && extra->rows > 0;
  if (has_x && (extra->N % 128 != 0 || extra->K % 64 != 0)) return cudaErrorInvalidValue;
  CUtensorMap ta, tg, tu, ta2, tg2, tu2;
  if (!make_tmap_bf16(&ta, A, a_rows, K, 128) ||
      !make_tmap_bf16(&tg, w_gate, static_cast<uint64_t>(G) * N, K, 128) ||
      !make_tmap_bf16(&tu, w_up, static_cast<uint64_t>(G) * N, K, 128))
    return cudaErrorInvalidValue;
  if (has_x) {
    if (!make_tmap_bf16(&ta2, extra->a, extra->rows, extra->K, 128) ||
        !make_tmap_bf16(&tg2, extra->w0, extra->N, extra->K, 128) ||
        !make_tmap_bf16(&tu2, extra->w1, extra->N, extra->K, 128))
      return cudaErrorInvalidValue;
  } else {
    ta2 = ta;  // never read without an extra group
    tg2 = tg;
    tu2 = tu;
  }
  DualParams dp{};
  if (has_x) {
    dp.x_rows = extra->rows;
    dp.x_N = extra->N;
    dp.x_K = extra->K;
    dp.x_out = extra->out;
    dp.x_ldo = extra->N;
  }
  dp.offsets = offsets;
  dp.counts = counts;
  dp.dense_rows = static_cast<int>(a_rows);  // used when offsets is null (one dense group)
  dp.G = offsets != nullptr ? G : 1;
  dp.K = K;
  dp.N = N;
  dp.masked_cap = masked_cap;
  dp.out = h;
  dp.ldo = N;
  dp.status = status;
  dp.next_item = counter;
  cudaError_t err = cudaMemsetAsync(counter, 0, sizeof(int32_t), st);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(tc_gemm_dual_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDualSmemBytes);
  if (err != cudaSuccess) return err;
  const long long max_items = ceil_div(a_rows, 128) * (N / 128) + (has_x ? ceil_div(extra->rows, 128) * (extra->N / 128) : 0);
  const long long sms = num_sms();
  const int grid = static_cast<int>(max_items < sms ? (max_items > 0 ? max_items : 1) : sms);
  trace_before(kid, st);
  err = launch_k(tc_gemm_dual_kernel<true>, grid, kDualThreads, kDualSmemBytes, st, ta, tg, tu, ta2, tg2, tu2, dp);
  trace_after(kid, st);
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t gemm_down_dual(const void* A, int64_t a_rows, const int32_t* offsets, const int32_t* counts, int G,
                           const void* w, int N, int K, void* y, int32_t* counter, int32_t* status, cudaStream_t st,
                           int masked_cap, bool y_f16, int kid, const DualExtra* extra) {
  if (G > kDualMaxGroups || N % 256 != 0 || K % 64 != 0) return cudaErrorInvalidValue;
  const bool has_x = extra != nullptr && extra->rows > 0;
  if (has_x && (extra->N % 256 != 0 || extra->K % 64 != 0)) return cudaErrorInvalidValue;
  CUtensorMap ta, tb, ta2, tb2;
  if (!make_tmap_bf16(&ta, A, a_rows, K, 128) || !make_tmap_bf16(&tb, w, static_cast<uint64_t>(G) * N, K, 256))
    return cudaErrorInvalidValue;
  if (has_x) {
    if (!make_tmap_bf16(&ta2, extra->a, extra->rows, extra->K, 128) ||
        !make_tmap_bf16(&tb2, extra->w0, extra->N, extra->K, 256))
      return cudaErrorInvalidValue;
  } else {
    ta2 = ta;  // never read without an extra group
    tb2 = tb;
  }
  DualParams dp{};
  if (has_x) {
    dp.x_rows = extra->rows;
    dp.x_N = extra->N;
    dp.x_K = extra->K;
    dp.x_out = extra->out;
    dp.x_ldo = extra->N;
  }
  dp.offsets = offsets;
  dp.counts = counts;
  dp.dense_rows = static_cast<int>(a_rows);  // used when offsets is null (one dense group)
  dp.G = offsets != nullptr ? G : 1;
  dp.K = K;
  dp.N = N;
  dp.masked_cap = masked_cap;
  dp.out = y;
  dp.ldo = N;
  dp.status = status;
  dp.next_item = counter;
  dp.out_f16 = y_f16 ? 1 : 0;
  cudaError_t err = cudaMemsetAsync(counter, 0, sizeof(int32_t), st);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(tc_gemm_dual_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDualSmemBytes);
  if (err != cudaSuccess) return err;
  const long long max_items = ceil_div(a_rows, 128) * (N / 256) + (has_x ? ceil_div(extra->rows, 128) * (extra->N / 256) : 0);
  const long long sms = num_sms();
  const int grid = static_cast<int>(max_items < sms ? (max_items > 0 ? max_items : 1) : sms);
  trace_before(kid, st);
  err = launch_k(tc_gemm_dual_kernel<false>, grid, kDualThreads, kDualSmemBytes, st, ta, tb, tb, ta2, tb2, tb2, dp);
  trace_after(kid, st);
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t gemm_down(const void* A, int64_t a_rows, const int32_t* offsets,
                      const int32_t* counts, int G, int dense_rows, const void* w, int N, int K,
                      float* y, int32_t* status, int kid, cudaStream_t st, int masked_cap) {
  CUtensorMap ta, tb;
  const bool wide = N % 256 == 0;
  if (!make_tmap_bf16(&ta, A, a_rows, K, 128) ||
      !make_tmap_bf16(&tb, w, static_cast<uint64_t>(G) * N, K, wide ? 256 : 128))
    return cudaErrorInvalidValue;
  GemmParams gp{};
  gp.offsets = offsets;
  gp.counts = counts;
  gp.G = G;
  gp.dense_rows = dense_rows;
  gp.K = K;
  gp.N = N;
  gp.b_rows_per_group = N;
  gp.out = y;
  gp.ldo = N;
  gp.status = status;
  gp.masked_cap = masked_cap;
  gp.half_tiles = 1;
  if (wide) {
    using Cfg = GemmCfg<256, EPI_F32, 4>;
    return launch<Cfg>(ta, tb, tb, gp, ceil_div(a_rows, 128) * ceil_div(N, 256), kid, st);
  }
  using Cfg = GemmCfg<128, EPI_F32, 6>;
  return launch<Cfg>(ta, tb, tb, gp, ceil_div(a_rows, 128) * ceil_div(N, 128), kid, st);
}

cudaError_t gemm_down_combine(const void* A, int64_t a_rows, const int32_t* offsets, const int32_t* counts,
                              int G, const void* w, int N, int K, const int32_t* pair_of_row,
                              const float* pair_weight, int topk, float* acc, int32_t* status, cudaStream_t st,
                              int masked_cap) {
  CUtensorMap ta, tb;
  const bool wide = N % 256 == 0;
  if (!make_tmap_bf16(&ta, A, a_rows, K, 128) ||
      !make_tmap_bf16(&tb, w, static_cast<uint64_t>(G) * N, K, wide ? 256 : 128))
    return cudaErrorInvalidValue;
  GemmParams gp{};
  gp.offsets = offsets;
  gp.counts = counts;
  gp.G = G;
  gp.dense_rows = 0;
  gp.K = K;
  gp.N = N;
  gp.b_rows_per_group = N;
  gp.out = acc;
  gp.ldo = N;
  gp.status = status;
  gp.pair_of_row = pair_of_row;
  gp.pair_weight = pair_weight;
  gp.topk = topk;
  gp.masked_cap = masked_cap;
  gp.half_tiles = 1;
  if (wide) {
    using Cfg = GemmCfg<256, EPI_COMBINE, 4>;
    return launch<Cfg>(ta, tb, tb, gp, ceil_div(a_rows, 128) * ceil_div(N, 256), MOE_K_DOWN, st);
  }
  using Cfg = GemmCfg<128, EPI_COMBINE, 6>;
  return launch<Cfg>(ta, tb, tb, gp, ceil_div(a_rows, 128) * ceil_div(N, 128), MOE_K_DOWN, st);
}

}  // namespace moe
