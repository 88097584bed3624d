// Host side of the two-SM (cta_group::2) expert GEMMs: tensor maps and cluster launches
// for bf16 (gate/up + SwiGLU, down with fp32 out) and block-scaled e4m3 (gate/up +
// SwiGLU + e4m3 re-quantisation, down with bf16 out).  Buckets must be 256-row aligned.
#include <cudaTypedefs.h>

#include "internal.h"
#include "tc_gemm_2cta.cuh"

namespace moe {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn2() {
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

// Rows of 128 bytes (64 bf16 or 128 e4m3) x box_rows, 128-byte swizzle.
bool tmap_rows128(CUtensorMap* m, const void* ptr, bool bytes, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn2();
  if (fn == nullptr) return false;
  const uint64_t esz = bytes ? 1 : 2;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * esz};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esz), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// n_atoms scale atoms of 512 bytes seen as [n_atoms, 128] 32-bit words; box = one atom.
bool tmap_atoms(CUtensorMap* m, const void* ptr, uint64_t n_atoms) {
  auto fn = encode_fn2();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {128, n_atoms};
  cuuint64_t strides[1] = {512};
  cuuint32_t box[2] = {128, 1};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

long long cdiv2(long long a, long long b) { return (a + b - 1) / b; }

template <class Cfg>
cudaError_t launch_pair(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                        const CUtensorMap& sfa, const CUtensorMap& sfb0, const CUtensorMap& sfb1,
                        const Pair2Params& pp, long long max_items, int kid, cudaStream_t st) {
  auto kern = tc_gemm_pair_kernel<Cfg>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  const long long clusters_max = num_sms() / 2;
  const long long clusters = max_items < clusters_max ? (max_items > 0 ? max_items : 1) : clusters_max;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * clusters), 1, 1);
  cfg.blockDim = dim3(Cfg::THREADS, 1, 1);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  trace_before(kid, st);
  err = cudaLaunchKernelEx(&cfg, kern, a, b0, b1, sfa, sfb0, sfb1, pp);
  trace_after(kid, st);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

Pair2Params pair_params(const int32_t* offsets, const int32_t* counts, int G, int K, int N, void* out,
                        uint8_t* out_sf, int32_t* status) {
  Pair2Params pp{};
  pp.offsets = offsets;
  pp.counts = counts;
  pp.G = G;
  pp.K = K;
  pp.N = N;
  pp.out = out;
  pp.ldo = N;
  pp.out_sf = out_sf;
  pp.status = status;
  return pp;
}

}  // namespace

cudaError_t gemm_pair_gateup_swiglu(const void* A, int64_t a_rows, const int32_t* offsets, const int32_t* counts,
                                    int G, const void* w_gate, const void* w_up, int N, int K, void* h,
                                    int32_t* status, cudaStream_t st) {
  using Cfg = Pair2Cfg<256, EPI2_SWIGLU_BF16, 6, false>;
  CUtensorMap ta, tg, tu;
  if (!tmap_rows128(&ta, A, false, a_rows, K, 128) ||
      !tmap_rows128(&tg, w_gate, false, static_cast<uint64_t>(G) * N, K, 128) ||
      !tmap_rows128(&tu, w_up, false, static_cast<uint64_t>(G) * N, K, 128))
    return cudaErrorInvalidValue;
  const Pair2Params pp = pair_params(offsets, counts, G, K, N, h, nullptr, status);
  return launch_pair<Cfg>(ta, tg, tu, ta, ta, ta, pp, cdiv2(a_rows, 256) * cdiv2(N, 128), MOE_K_GATEUP, st);
}

cudaError_t gemm_pair_down(const void* A, int64_t a_rows, const int32_t* offsets, const int32_t* counts, int G,
                           const void* w, int N, int K, float* y, int32_t* status, cudaStream_t st) {
  using Cfg = Pair2Cfg<256, EPI2_F32, 6, false>;
  CUtensorMap ta, tb;
  if (!tmap_rows128(&ta, A, false, a_rows, K, 128) ||
      !tmap_rows128(&tb, w, false, static_cast<uint64_t>(G) * N, K, 128))
    return cudaErrorInvalidValue;
  const Pair2Params pp = pair_params(offsets, counts, G, K, N, y, nullptr, status);
  return launch_pair<Cfg>(ta, tb, tb, ta, ta, ta, pp, cdiv2(a_rows, 256) * cdiv2(N, 256), MOE_K_DOWN, st);
}

cudaError_t gemm_pair_gateup_swiglu_fp8(const void* A, const uint8_t* a_atoms, int64_t a_rows,
                                        const int32_t* offsets, const int32_t* counts, int G, const void* w_gate,
                                        const void* w_up, const uint8_t* gate_atoms, const uint8_t* up_atoms,
                                        int N, int K, void* h, uint8_t* h_atoms, int32_t* status,
                                        cudaStream_t st) {
  using Cfg = Pair2Cfg<256, EPI2_SWIGLU_E4M3, 6, true>;
  const uint64_t m_tiles = static_cast<uint64_t>(cdiv2(a_rows, 256) * 2);
  const uint64_t kb4 = (K / 128 + 3) / 4;
  const uint64_t w_atoms = static_cast<uint64_t>(G) * (N / 128) * kb4;
  CUtensorMap ta, tg, tu, tsa, tsg, tsu;
  if (!tmap_rows128(&ta, A, true, a_rows, K, 128) ||
      !tmap_rows128(&tg, w_gate, true, static_cast<uint64_t>(G) * N, K, 128) ||
      !tmap_rows128(&tu, w_up, true, static_cast<uint64_t>(G) * N, K, 128) ||
      !tmap_atoms(&tsa, a_atoms, m_tiles * kb4) || !tmap_atoms(&tsg, gate_atoms, w_atoms) ||
      !tmap_atoms(&tsu, up_atoms, w_atoms))
    return cudaErrorInvalidValue;
  const Pair2Params pp = pair_params(offsets, counts, G, K, N, h, h_atoms, status);
  return launch_pair<Cfg>(ta, tg, tu, tsa, tsg, tsu, pp, cdiv2(a_rows, 256) * cdiv2(N, 128), MOE_K_GATEUP, st);
}

cudaError_t gemm_pair_down_fp8(const void* A, const uint8_t* a_atoms, int64_t a_rows, const int32_t* offsets,
                               const int32_t* counts, int G, const void* w, const uint8_t* w_atoms, int N, int K,
                               void* y, int32_t* status, cudaStream_t st) {
  using Cfg = Pair2Cfg<128, EPI2_BF16, 8, true>;
  const uint64_t m_tiles = static_cast<uint64_t>(cdiv2(a_rows, 256) * 2);
  const uint64_t kb4 = (K / 128 + 3) / 4;
  const uint64_t n_w_atoms = static_cast<uint64_t>(G) * (N / 128) * kb4;
  CUtensorMap ta, tb, tsa, tsb;
  if (!tmap_rows128(&ta, A, true, a_rows, K, 128) ||
      !tmap_rows128(&tb, w, true, static_cast<uint64_t>(G) * N, K, 64) ||
      !tmap_atoms(&tsa, a_atoms, m_tiles * kb4) || !tmap_atoms(&tsb, w_atoms, n_w_atoms))
    return cudaErrorInvalidValue;
  const Pair2Params pp = pair_params(offsets, counts, G, K, N, y, nullptr, status);
  return launch_pair<Cfg>(ta, tb, tb, tsa, tsb, tsb, pp, cdiv2(a_rows, 256) * cdiv2(N, 128), MOE_K_DOWN, st);
}

}  // namespace moe
