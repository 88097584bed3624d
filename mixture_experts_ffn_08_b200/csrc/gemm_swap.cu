// Host side of the swap-A/B gate/up for e2m1 expert weights (tc_gemm_swap.cuh), and the
// two small kernels it needs: the token-tile schedule and the tokens' padded scale atoms.
#include <cudaTypedefs.h>

#include "internal.h"
#include "tc_gemm_swap.cuh"

namespace moe {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn_swap() {
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

// Row-major matrix [rows, cols] of 1-byte values (e4m3) or packed e2m1 (cols 4-bit values,
// unpacked by the TMA to one byte per value in shared memory), box of 128 columns x
// box_rows rows, 128-byte swizzle.
bool make_tmap_swap(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
                    bool e2m1) {
  auto fn = encode_fn_swap();
  if (fn == nullptr || cols % 128 != 0) return false;
  if (e2m1 && (reinterpret_cast<uintptr_t>(ptr) & 31) != 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {e2m1 ? cols / 2 : cols};
  cuuint32_t box[2] = {128, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, e2m1 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
            const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

constexpr int kTokTile = SwapCfg::BT;

// tsched[e] = sum over j < e of ceil(counts[j] / 32), tsched[E] = the total (one block, E <= 1024).
__global__ void __launch_bounds__(1024) token_tile_schedule_kernel(const int32_t* __restrict__ counts, int E,
                                                                   int32_t* __restrict__ tsched) {
  __shared__ int warp_tot[32];
  const int e = threadIdx.x, lane = e & 31, w = e >> 5;
  const int tiles = e < E ? (__ldg(counts + e) + kTokTile - 1) / kTokTile : 0;
  int v = tiles;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[w] = v;
  __syncthreads();
  if (w == 0) {
    int t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += n;
    }
    warp_tot[lane] = t;  // inclusive totals of warps 0..lane
  }
  __syncthreads();
  const int incl = v + (w > 0 ? warp_tot[w - 1] : 0);
  if (e < E) tsched[e] = incl - tiles;
  if (e == E - 1) tsched[E] = incl;
}

// Tokens' scales [rows, nk] fp32 (powers of two) -> padded atoms [token tiles][ceil(nk/4)][512]:
// row t (16 bytes) of atom (v, q) holds, in each of its four words, the UE8M0 scales of
// token t of tile v for K steps 4q..4q+3 (byte b = step 4q+b; 127, a scale of 1, past nk).
__global__ void swap_token_atoms_kernel(const float* __restrict__ scales, int nk,
                                        const int32_t* __restrict__ offsets,
                                        const int32_t* __restrict__ tsched, int G,
                                        uint8_t* __restrict__ atoms) {
  const int nk4 = (nk + 3) / 4;
  const long long n = static_cast<long long>(__ldg(tsched + G)) * nk4 * kTokTile;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const int t = static_cast<int>(i % kTokTile);
    const long long a = i / kTokTile;  // atom (v, q)
    const int q = static_cast<int>(a % nk4);
    const int v = static_cast<int>(a / nk4);
    int lo = 0, hi = G - 1;  // expert of token tile v: smallest g with tsched[g+1] > v
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(tsched + mid + 1) > v) hi = mid; else lo = mid + 1;
    }
    const long long row = __ldg(offsets + lo) + static_cast<long long>(v - __ldg(tsched + lo)) * kTokTile + t;
    uint32_t w = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int kb = 4 * q + b;
      const uint32_t e = kb < nk ? (__float_as_uint(__ldg(scales + row * nk + kb)) >> 23) & 0xFFu : 127u;
      w |= e << (8 * b);
    }
    reinterpret_cast<uint4*>(atoms)[i] = make_uint4(w, w, w, w);
  }
}

long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

}  // namespace

long long swap_max_token_tiles(long long pairs, int E) { return cdiv(pairs, kTokTile) + E; }

cudaError_t gemm_gateup_swiglu_swap(const void* x_perm, const float* x_scale, int64_t x_rows,
                                    const int32_t* offsets, const int32_t* counts, int G,
                                    long long max_tiles, const void* w_gate, const void* w_up,
                                    const uint8_t* gate_atoms, const uint8_t* up_atoms, int N, int K,
                                    void* h, uint8_t* h_atoms, int32_t* tsched, uint8_t* tok_atoms,
                                    int32_t* status, cudaStream_t st) {
  if (G > 1024 || N % 128 != 0 || K % 128 != 0) return cudaErrorInvalidValue;
  CUtensorMap tg, tu, tx;
  if (!make_tmap_swap(&tg, w_gate, static_cast<uint64_t>(G) * N, K, 128, true) ||
      !make_tmap_swap(&tu, w_up, static_cast<uint64_t>(G) * N, K, 128, true) ||
      !make_tmap_swap(&tx, x_perm, x_rows, K, kTokTile, false))
    return cudaErrorInvalidValue;
  cudaError_t err;
  trace_before(MOE_K_SCALE_ATOMS, st);
  token_tile_schedule_kernel<<<1, 1024, 0, st>>>(counts, G, tsched);
  trace_after(MOE_K_SCALE_ATOMS, st);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const int nk = K / 128;
  const long long n_atoms = max_tiles * cdiv(nk, 4) * kTokTile;
  const long long ab = cdiv(n_atoms, 256);
  const int agrid = static_cast<int>(ab < num_sms() * 8LL ? (ab > 0 ? ab : 1) : num_sms() * 8LL);
  trace_before(MOE_K_SCALE_ATOMS, st);
  swap_token_atoms_kernel<<<agrid, 256, 0, st>>>(x_scale, nk, offsets, tsched, G, tok_atoms);
  trace_after(MOE_K_SCALE_ATOMS, st);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;

  SwapParams sp{};
  sp.offsets = offsets;
  sp.counts = counts;
  sp.tsched = tsched;
  sp.G = G;
  sp.K = K;
  sp.N = N;
  sp.sfw0 = gate_atoms;
  sp.sfw1 = up_atoms;
  sp.sft = tok_atoms;
  sp.out = static_cast<uint8_t*>(h);
  sp.out_sf = h_atoms;
  sp.status = status;
  auto kern = tc_gemm_swap_kernel<SwapCfg>;
  if ((err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SwapCfg::SMEM_BYTES)) !=
      cudaSuccess)
    return err;
  const long long items = max_tiles * (N / 128);
  const long long sms = num_sms();
  const int grid = static_cast<int>(items < sms ? (items > 0 ? items : 1) : sms);
  trace_before(MOE_K_GATEUP, st);
  kern<<<grid, SwapCfg::THREADS, SwapCfg::SMEM_BYTES, st>>>(tg, tu, tx, sp);
  trace_after(MOE_K_GATEUP, st);
  return cudaGetLastError();
}

}  // namespace moe
