// Internal launchers shared between the translation units of the library.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kBlockM = 128;    // M-tile of the one-SM grouped GEMM (bucket alignment)
constexpr int kBlockM2 = 256;   // bucket alignment for the two-SM (cta_group::2) GEMMs
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;
constexpr int kPermChunk = 256;  // pairs per chunk of the stable bucket ranking
constexpr int kSmallPairs = 2048;  // up to this many pairs one block counts, scans and ranks

// Programmatic dependent launch of the layer's kernels (api.cu): on unless the
// environment sets MOE_DISABLE_PDL to a non-empty value other than "0".
bool pdl_enabled();

// Launches kern<<<grid, block, smem, st>>>(args...) with programmatic stream
// serialization when pdl_enabled(); every kernel launched this way calls pdl_wait()
// before it reads or writes global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// K-slices of the router GEMM.  With few output tiles (small T) the reduction over H is
// split so that about 128 CTAs work; slice s writes its own fp32 partial logits at
// s * T * E, and the top-k kernel adds the slices in order s = 0, 1, ... (the same sum
// on every run).  At least 4 K-blocks of 64 per slice.
inline int router_k_splits(long long T, int H, int E) {
  const long long tiles = ((T + 127) / 128) * ((E + 255) / 256);
  const long long kb = H / 64;
  long long s = tiles > 0 ? 128 / tiles : 1;
  if (s > kb / 4) s = kb / 4;
  return s < 1 ? 1 : static_cast<int>(s);
}

// Tracing (api.cu): brackets a launch of kernel `kid` with events when enabled.
void trace_before(int kid, cudaStream_t st);
void trace_after(int kid, cudaStream_t st);
int num_sms();

// Activations (x, h) are e4m3 with 1x128 scales: the FP8 and the FP8 x FP4 layers.
inline bool act_e4m3(const moe_params_t& p) {
  return p.dtype == MOE_DTYPE_FP8_E4M3 || p.dtype == MOE_DTYPE_FP8_FP4;
}

// ---------------------------------------------------------------- routing (kernels.cu)
cudaError_t launch_dequant_x(const uint8_t* xq, const float* xs, int T, int H, void* x_bf16,
                             cudaStream_t st);
// logits: n_part slices of [T, E] fp32 partial sums, summed in slice order.
cudaError_t launch_topk(const float* logits, const moe_params_t& p, const float* bias,
                        int32_t* ids, float* w, cudaStream_t st, int n_part = 1);

// b_e += gamma * sign(mean load - load_e) (aux-free balancing bias).
cudaError_t launch_bias_update(const int32_t* counts, int E, float gamma, float* bias, cudaStream_t st);

// ---------------------------------------------------------------- dispatch (kernels.cu)
// Masked layout with a compact GEMM schedule: with masked_cap > 0 the grouped GEMMs take
// `offsets` as the schedule, the 128-padded prefix sums of counts (masked_schedule), and
// address group g's rows at g * masked_cap.
cudaError_t launch_masked_schedule(const int32_t* counts, int E, int32_t* sched, cudaStream_t st);
// One CTA waits on an mbarrier nothing completes, for limit_ns, then sets MOE_DEV_TIMEOUT.
cudaError_t launch_bounded_wait_selftest(int32_t* status, long long limit_ns, cudaStream_t st);
// offsets[e] = e * cap for e in [0, E] (masked layout row ranges).
cudaError_t launch_masked_offsets(int E, int cap, int32_t* offsets, cudaStream_t st);
// fill_pad: the moe_permute contract: contiguous layout, zero the pad rows of x_perm (scale 1
// for FP8); both layouts, pair_of_row = -1 on rows without a pair.  The layer itself passes
// false: its GEMMs never store a pad row and an MMA row depends on its own A row only, so
// whatever the pad rows hold stays in rows nobody reads; x is then copied token by token
// (each x row read once) instead of row by row.
cudaError_t launch_permute(const moe_params_t& p, int block_m, const int32_t* ids, const void* x,
                           const float* x_scale, int32_t* counts, int32_t* offsets,
                           int32_t* row_of_pair, int32_t* pair_of_row, void* x_perm,
                           float* x_perm_scale, int32_t* chunk_counts, int32_t* status,
                           cudaStream_t st, bool fill_pad = true, uint8_t* x_atoms = nullptr);

// ---------------------------------------------------------------- combine (kernels.cu)
// y_perm is fp32 for bf16 workloads and bf16 for FP8 workloads (p.dtype).
// y_shared: [T,H] fp32, or fp16 when ysh_f16.
cudaError_t launch_combine(const moe_params_t& p, const void* y_perm, const int32_t* row_of_pair,
                           const float* w, const void* y_shared, void* out, cudaStream_t st, bool y_f16 = false,
                           bool ysh_f16 = false);

// ---------------------------------------------------------------- GEMMs (gemm.cu)
// Router logits x [T,H] bf16 @ W_r[E,H]^T as router_k_splits(T, H, E) fp32 partial
// slices [T, E], slice s at logits + s*T*E.
cudaError_t gemm_router(const void* x, const void* w_r, int T, int H, int E, float* logits,
                        int32_t* status, cudaStream_t st);
// h [rows, N] bf16 = SiLU(A Wg^T) * (A Wu^T), grouped by offsets (or dense when null);
// with counts, pad rows of each group are not stored.
cudaError_t gemm_gateup_swiglu(const void* A, int64_t a_rows, const int32_t* offsets,
                               const int32_t* counts, int G, int dense_rows, const void* w_gate,
                               const void* w_up, int N, int K, void* h, int32_t* status, int kid,
                               cudaStream_t st, int masked_cap = 0);
// The same gate/up projection with two M-tiles of an expert per work item (grouped, with
// counts, N multiple of 128); counter is a device int the call zeroes before the launch.
// offsets == nullptr: one dense group of a_rows rows (counts unused).
// An extra dense group for the two-tile launches (the shared expert): A [rows, K] bf16,
// weights [N, K] bf16 (w1: the up projection's, for gate/up), output [rows, N] stored like
// the launch's own (h bf16; y fp16 or fp32 as the launch's y_f16 says).
struct DualExtra {
  const void* a;
  int rows;
  const void* w0;
  const void* w1;
  int N;
  int K;
  void* out;
};
cudaError_t gemm_gateup_swiglu_dual(const void* A, int64_t a_rows, const int32_t* offsets, const int32_t* counts,
                                    int G, const void* w_gate, const void* w_up, int N, int K, void* h,
                                    int32_t* counter, int32_t* status, cudaStream_t st, int masked_cap = 0,
                                    int kid = MOE_K_GATEUP, const DualExtra* extra = nullptr);
// The down projection with two M-tiles per work item (N multiple of 256); counter as above.
cudaError_t gemm_down_dual(const void* A, int64_t a_rows, const int32_t* offsets, const int32_t* counts, int G,
                           const void* w, int N, int K, void* y, int32_t* counter, int32_t* status, cudaStream_t st,
                           int masked_cap = 0, bool y_f16 = false, int kid = MOE_K_DOWN,
                           const DualExtra* extra = nullptr);
// y [rows, N] fp32 = A W^T, grouped by offsets (or dense when null); with counts, pad
// rows of each group are not stored.
cudaError_t gemm_down(const void* A, int64_t a_rows, const int32_t* offsets,
                      const int32_t* counts, int G, int dense_rows, const void* w, int N, int K,
                      float* y, int32_t* status, int kid, cudaStream_t st, int masked_cap = 0);

// acc[t] += w[p] * (A W^T)[r] for every bucket row r of pair p = pair_of_row[r], t = p / topk
// (down projection fused with the combine; fp32 vector reductions, order not fixed).
cudaError_t gemm_down_combine(const void* A, int64_t a_rows, const int32_t* offsets, const int32_t* counts,
                              int G, const void* w, int N, int K, const int32_t* pair_of_row,
                              const float* pair_weight, int topk, float* acc, int32_t* status, cudaStream_t st,
                              int masked_cap = 0);
// out[i] = bf16(acc[i]) for n values (n multiple of 8).
cudaError_t launch_f32_to_bf16(const float* acc, long long n, void* out, cudaStream_t st);

// ---------------------------------------------------------------- FP8 GEMMs (gemm_fp8.cu)
// fp32 power-of-two scales -> 512-byte UE8M0 scale atoms (see tc_gemm_fp8.cuh).
cudaError_t launch_sf_rows_to_atoms(const float* scales, int nk, const int32_t* offsets, int G,
                                    long long max_rows, uint8_t* atoms, cudaStream_t st);
cudaError_t launch_sf_blocks_to_atoms(const float* scales, long long nblk, int nk, uint8_t* atoms,
                                      cudaStream_t st);
// h (e4m3 [rows, N] + scale atoms) = quant(SiLU(A Wg^T) * (A Wu^T)), block-scaled e4m3 GEMM.
cudaError_t gemm_gateup_swiglu_fp8(const void* A, const uint8_t* a_atoms, int64_t a_rows,
                                   const int32_t* offsets, const int32_t* counts, int G,
                                   const void* w_gate, const void* w_up, const uint8_t* gate_atoms,
                                   const uint8_t* up_atoms, int N, int K, void* h, uint8_t* h_atoms,
                                   int32_t* status, cudaStream_t st, int masked_cap = 0, bool w4 = false);
// y [rows, N] bf16 = A W^T, block-scaled e4m3 GEMM.
cudaError_t gemm_down_fp8(const void* A, const uint8_t* a_atoms, int64_t a_rows,
                          const int32_t* offsets, const int32_t* counts, int G, const void* w,
                          const uint8_t* w_atoms, int N, int K, void* y, int32_t* status,
                          cudaStream_t st, int masked_cap = 0, bool w4 = false);
// w4: weights are packed e2m1 (cols/2 bytes per row, 32-byte aligned base) and the weight
// atoms come from launch_fp4_scale_atoms.
// e2m1 weight scale words [rows, K/128] (4 UE8M0 bytes each) -> atoms [rows/128][K/128][512].
cudaError_t launch_fp4_scale_atoms(const uint32_t* words, long long rows, int K, uint8_t* atoms, cudaStream_t st);

// ---------------------------------------------------------------- two-SM GEMMs (gemm_2cta.cu)
cudaError_t gemm_pair_gateup_swiglu(const void* A, int64_t a_rows, const int32_t* offsets, const int32_t* counts,
                                    int G, const void* w_gate, const void* w_up, int N, int K, void* h,
                                    int32_t* status, cudaStream_t st);
cudaError_t gemm_pair_down(const void* A, int64_t a_rows, const int32_t* offsets, const int32_t* counts, int G,
                           const void* w, int N, int K, float* y, int32_t* status, cudaStream_t st);
cudaError_t gemm_pair_gateup_swiglu_fp8(const void* A, const uint8_t* a_atoms, int64_t a_rows,
                                        const int32_t* offsets, const int32_t* counts, int G, const void* w_gate,
                                        const void* w_up, const uint8_t* gate_atoms, const uint8_t* up_atoms,
                                        int N, int K, void* h, uint8_t* h_atoms, int32_t* status,
                                        cudaStream_t st);
cudaError_t gemm_pair_down_fp8(const void* A, const uint8_t* a_atoms, int64_t a_rows, const int32_t* offsets,
                               const int32_t* counts, int G, const void* w, const uint8_t* w_atoms, int N, int K,
                               void* y, int32_t* status, cudaStream_t st);

}  // namespace moe
