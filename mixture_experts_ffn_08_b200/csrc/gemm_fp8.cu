// Host side of the block-scaled FP8 expert GEMMs, and the kernels that turn the layer's
// fp32 power-of-two block scales into the 512-byte UE8M0 scale atoms the tensor core
// reads (layout described in tc_gemm_fp8.cuh).
#include <cudaTypedefs.h>

#include "internal.h"
#include "tc_gemm_fp8.cuh"

namespace moe {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn8() {
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

// Row-major byte matrix [rows, cols], box of 128 columns (128 bytes) x box_rows rows,
// 128-byte swizzle; out-of-range rows read as zero.
bool make_tmap_u8(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn8();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed e2m1 matrix [rows, cols] (cols 4-bit values, cols/2 bytes per row), box of 128
// values x box_rows rows; TMA unpacks every 16 values (8 bytes) into a 16-byte smem slot,
// so the box lands as 128 bytes per row under the 128-byte swizzle, like an e4m3 box.
// Needs a 32-byte aligned base and cols a multiple of 128.
bool make_tmap_e2m1(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn8();
  if (fn == nullptr || (reinterpret_cast<uintptr_t>(ptr) & 31) != 0 || cols % 128 != 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols / 2};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_w(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows, bool w4) {
  return w4 ? make_tmap_e2m1(m, ptr, rows, cols, box_rows) : make_tmap_u8(m, ptr, rows, cols, box_rows);
}

template <class Cfg>
cudaError_t launch8(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                    const Fp8Params& fp, long long max_items, int kid, cudaStream_t st) {
  auto kern = tc_gemm_fp8_kernel<Cfg>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
  if (err != cudaSuccess) return err;
  const long long sms = num_sms();
  const int grid = static_cast<int>(max_items < sms ? (max_items > 0 ? max_items : 1) : sms);
  trace_before(kid, st);
  err = launch_k(kern, grid, Cfg::THREADS, Cfg::SMEM_BYTES, st, a, b0, b1, fp);
  trace_after(kid, st);
  return err != cudaSuccess ? err : cudaGetLastError();
}

// UE8M0 byte of a power-of-two fp32 scale: its biased exponent field.
__device__ __forceinline__ uint32_t ue8m0_of(float s) { return (__float_as_uint(s) >> 23) & 0xFFu; }

// Per-row scales [rows, nk] (one per 128 columns) -> atoms [rows/128][ceil(nk/4)][512]:
// scale kb of row r is byte kb % 4 of the row's word in atom kb / 4.  For the rows of the
// buckets (offsets[G] of them).
__global__ void sf_rows_to_atoms_kernel(const float* __restrict__ scales, int nk,
                                        const int32_t* __restrict__ offsets, int G,
                                        uint8_t* __restrict__ atoms) {
  pdl_launch_dependents();
  pdl_wait();
  const long long n = static_cast<long long>(__ldg(offsets + G)) * nk;
  const int nk4 = (nk + 3) / 4;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / nk;
    const int kb = static_cast<int>(i % nk);
    uint8_t* atom = atoms + ((r >> 7) * nk4 + (kb >> 2)) * 512;
    atom[sf_atom_offset(static_cast<int>(r & 127)) + (kb & 3)] = static_cast<uint8_t>(ue8m0_of(__ldg(scales + i)));
  }
}

// One scale per 128x128 weight block, blocks [nblk][nk] -> atoms [nblk][ceil(nk/4)][512]
// whose 128 words all hold the scales of four consecutive K blocks.
__global__ void sf_blocks_to_atoms_kernel(const float* __restrict__ scales, long long nblk, int nk,
                                          uint8_t* __restrict__ atoms) {
  pdl_launch_dependents();
  pdl_wait();
  const int nk4 = (nk + 3) / 4;
  const long long n = nblk * nk4 * 32;  // 32 x 16 bytes per atom
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long a = i >> 5;
    const long long blk = a / nk4;
    const int kb0 = static_cast<int>(a % nk4) * 4;
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t b = kb0 + j < nk ? ue8m0_of(__ldg(scales + blk * nk + kb0 + j)) : 127u;
      w |= b << (8 * j);
    }
    reinterpret_cast<uint4*>(atoms)[i] = make_uint4(w, w, w, w);
  }
}

long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

}  // namespace

cudaError_t launch_sf_rows_to_atoms(const float* scales, int nk, const int32_t* offsets, int G,
                                    long long max_rows, uint8_t* atoms, cudaStream_t st) {
  const long long n = max_rows * nk;
  const int grid = static_cast<int>(cdiv(n, 256) < num_sms() * 8LL ? cdiv(n, 256) : num_sms() * 8LL);
  trace_before(MOE_K_SCALE_ATOMS, st);
  const cudaError_t err = launch_k(sf_rows_to_atoms_kernel, grid > 0 ? grid : 1, 256, 0, st, scales, nk, offsets, G, atoms);
  trace_after(MOE_K_SCALE_ATOMS, st);
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_sf_blocks_to_atoms(const float* scales, long long nblk, int nk, uint8_t* atoms,
                                      cudaStream_t st) {
  const long long n = nblk * ((nk + 3) / 4) * 32;
  const int grid = static_cast<int>(cdiv(n, 256) < num_sms() * 8LL ? cdiv(n, 256) : num_sms() * 8LL);
  trace_before(MOE_K_SCALE_ATOMS, st);
  const cudaError_t err = launch_k(sf_blocks_to_atoms_kernel, grid > 0 ? grid : 1, 256, 0, st, scales, nblk, nk, atoms);
  trace_after(MOE_K_SCALE_ATOMS, st);
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t gemm_gateup_swiglu_fp8(const void* A, const uint8_t* a_atoms, int64_t a_rows,
                                   const int32_t* offsets, const int32_t* counts, int G,
                                   const void* w_gate, const void* w_up, const uint8_t* gate_atoms,
                                   const uint8_t* up_atoms, int N, int K, void* h, uint8_t* h_atoms,
                                   int32_t* status, cudaStream_t st, int masked_cap, bool w4) {
  CUtensorMap ta, tg, tu;
  if (!make_tmap_u8(&ta, A, a_rows, K, 128) ||
      !make_tmap_w(&tg, w_gate, static_cast<uint64_t>(G) * N, K, 128, w4) ||
      !make_tmap_w(&tu, w_up, static_cast<uint64_t>(G) * N, K, 128, w4))
    return cudaErrorInvalidValue;
  Fp8Params fp{};
  fp.offsets = offsets;
  fp.counts = counts;
  fp.G = G;
  fp.K = K;
  fp.N = N;
  fp.sfa = a_atoms;
  fp.sfb0 = gate_atoms;
  fp.sfb1 = up_atoms;
  fp.out = h;
  fp.ldo = N;
  fp.out_sf = h_atoms;
  fp.status = status;
  fp.masked_cap = masked_cap;
  const long long items = cdiv(a_rows, 128) * cdiv(N, 128);
  if (w4) return launch8<Fp8Cfg<256, EPI8_SWIGLU_Q, 4, true>>(ta, tg, tu, fp, items, MOE_K_GATEUP, st);
  return launch8<Fp8Cfg<256, EPI8_SWIGLU_Q, 4>>(ta, tg, tu, fp, items, MOE_K_GATEUP, st);
}

cudaError_t gemm_down_fp8(const void* A, const uint8_t* a_atoms, int64_t a_rows,
                          const int32_t* offsets, const int32_t* counts, int G, const void* w,
                          const uint8_t* w_atoms, int N, int K, void* y, int32_t* status,
                          cudaStream_t st, int masked_cap, bool w4) {
  // 256-column tiles (one accumulator) read A half as often per output as 128-column
  // ones; they need whole 256-row weight slices, so N % 256 == 0.
  const bool wide = N % 256 == 0;
  CUtensorMap ta, tb;
  if (!make_tmap_u8(&ta, A, a_rows, K, 128) ||
      !make_tmap_w(&tb, w, static_cast<uint64_t>(G) * N, K, wide ? 256 : 128, w4))
    return cudaErrorInvalidValue;
  Fp8Params fp{};
  fp.offsets = offsets;
  fp.counts = counts;
  fp.G = G;
  fp.K = K;
  fp.N = N;
  fp.sfa = a_atoms;
  fp.sfb0 = w_atoms;
  fp.sfb1 = nullptr;
  fp.out = y;
  fp.ldo = N;
  fp.out_sf = nullptr;
  fp.status = status;
  fp.masked_cap = masked_cap;
  const long long rows = cdiv(a_rows, 128);
  if (wide) {
    if (w4) return launch8<Fp8Cfg<256, EPI8_BF16, 4, true>>(ta, tb, tb, fp, rows * cdiv(N, 256), MOE_K_DOWN, st);
    return launch8<Fp8Cfg<256, EPI8_BF16, 4>>(ta, tb, tb, fp, rows * cdiv(N, 256), MOE_K_DOWN, st);
  }
  if (w4) return launch8<Fp8Cfg<128, EPI8_BF16, 5, true>>(ta, tb, tb, fp, rows * cdiv(N, 128), MOE_K_DOWN, st);
  return launch8<Fp8Cfg<128, EPI8_BF16, 5>>(ta, tb, tb, fp, rows * cdiv(N, 128), MOE_K_DOWN, st);
}

// e2m1 weight scales: word (row r, K step kb) of the caller's [rows, K/128] words (byte j
// = UE8M0 scale of K elements 128 kb + 32 j ...) goes to atom (r / 128, kb) at the
// position of row r % 128.
__global__ void fp4_scale_atoms_kernel(const uint32_t* __restrict__ words, long long rows, int kb_n,
                                       uint8_t* __restrict__ atoms) {
  const long long n = rows * kb_n;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long r = i / kb_n;
    const int kb = static_cast<int>(i % kb_n);
    uint8_t* atom = atoms + ((r >> 7) * kb_n + kb) * 512;
    *reinterpret_cast<uint32_t*>(atom + sf_atom_offset(static_cast<int>(r & 127))) = __ldg(words + i);
  }
}

cudaError_t launch_fp4_scale_atoms(const uint32_t* words, long long rows, int K, uint8_t* atoms, cudaStream_t st) {
  const long long n = rows * (K / 128);
  const long long blocks = cdiv(n, 256);
  const int grid = static_cast<int>(blocks < num_sms() * 8LL ? (blocks > 0 ? blocks : 1) : num_sms() * 8LL);
  fp4_scale_atoms_kernel<<<grid, 256, 0, st>>>(words, rows, K / 128, atoms);
  return cudaGetLastError();
}

}  // namespace moe
